"""ctypes wrapper around the C++ oracle (test infrastructure only).

Every function here forwards to ``loopkv_oracle.cpp``; nothing is computed in
Python beyond array allocation.  Arrays of bf16 values travel as their raw
16-bit patterns (``numpy.uint16``).
"""

import ctypes
import dataclasses

import numpy as np

from . import build as _build

KIND_Q4, KIND_Q2, KIND_SHARE, KIND_BF16, KIND_RES2 = 0, 1, 2, 3, 4
G = 32

_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(_build.build())
    P = ctypes.c_void_p
    lib.orc_quantize_group.argtypes = [P, ctypes.c_int, P, P, P]
    lib.orc_quantize_group.restype = None
    lib.orc_unit_new.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.orc_unit_new.restype = P
    lib.orc_unit_free.argtypes = [P]
    lib.orc_unit_free.restype = None
    lib.orc_unit_len.argtypes = [P]
    lib.orc_unit_len.restype = ctypes.c_int
    lib.orc_unit_append.argtypes = [P, P, P, ctypes.c_int]
    lib.orc_unit_append.restype = ctypes.c_int
    lib.orc_unit_export.argtypes = [P, P, P, P, P, P, P, P]
    lib.orc_unit_export.restype = ctypes.c_int
    lib.orc_region_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.orc_region_bytes.restype = ctypes.c_size_t
    lib.orc_unit_serialize.argtypes = [P, P, P, P, ctypes.c_size_t]
    lib.orc_unit_serialize.restype = ctypes.c_int
    lib.orc_decode.argtypes = [P, P, P, ctypes.c_double, ctypes.c_double,
                               ctypes.c_double, P, P, P, P, P, P, P]
    lib.orc_decode.restype = ctypes.c_int
    lib.orc_decode_group.argtypes = [P, P, P, ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                     ctypes.c_double, P, P, P, P, P, P, P]
    lib.orc_decode_group.restype = ctypes.c_int
    lib.orc_vq_decode.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_int, P, P, P, P, P, ctypes.c_double, P, P]
    lib.orc_vq_decode.restype = ctypes.c_int
    lib.orc_vq_encode.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P]
    lib.orc_vq_encode.restype = ctypes.c_int
    lib.orc_plan_brute.argtypes = [ctypes.c_int, ctypes.c_int, P, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_int, P, P, P, P]
    lib.orc_plan_brute.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def quantize_group(x, bits):
    """Quantize 32 fp32 values at ``bits`` (4 or 2) -> (codes u8[32], scale, zero)."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    assert x.shape == (G,)
    code = np.zeros(G, np.uint8)
    scale = np.zeros(1, np.float32)
    zero = np.zeros(1, np.float32)
    lib.orc_quantize_group(_ptr(x), bits, _ptr(code), _ptr(scale), _ptr(zero))
    return code, scale[0], zero[0]


def region_bytes(kind, D, cap):
    """Bytes of one unit's region in the canonical cache layout."""
    return int(_load().orc_region_bytes(kind, D, cap))


class OracleUnit:
    """One (cell, sequence, head) unit: its cache state after appends."""

    def __init__(self, kind, D, cap):
        lib = _load()
        self._lib = lib  # free with the library that made the handle
        self._h = lib.orc_unit_new(kind, D, cap)
        if not self._h:
            raise ValueError("bad unit kind=%r D=%r cap=%r" % (kind, D, cap))
        self.kind, self.D, self.cap = kind, D, cap

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            self._lib.orc_unit_free(h)
            self._h = None

    @property
    def n(self):
        return int(self._lib.orc_unit_len(self._h))

    def append(self, k_bits, v_bits):
        """Append tokens given as bf16 bit patterns of shape [n_new, D]."""
        k = np.ascontiguousarray(k_bits, dtype=np.uint16).reshape(-1, self.D)
        v = np.ascontiguousarray(v_bits, dtype=np.uint16).reshape(-1, self.D)
        assert k.shape == v.shape
        rc = self._lib.orc_unit_append(self._h, _ptr(k), _ptr(v), k.shape[0])
        if rc != 0:
            raise ValueError("oracle append rejected (capacity)")

    def export(self, src=None):
        """Quantized state: dict of key/value codes, scales and zero points.

        ``src``: the reference unit of a residual (RES2) unit, whose codes are
        its residual codes against that reference.
        """
        sh = None if src is None else src._h
        qtok = self._lib.orc_unit_export(self._h, sh, None, None, None, None, None, None)
        if qtok < 0:
            raise ValueError("residual unit without a reference holding its positions")
        D = self.D
        kq = np.zeros((qtok, D), np.uint8)
        ks = np.zeros((qtok // G, D), np.float32)
        kz = np.zeros((qtok // G, D), np.float32)
        vq = np.zeros((qtok, D), np.uint8)
        vs = np.zeros((qtok, D // G), np.float32)
        vz = np.zeros((qtok, D // G), np.float32)
        self._lib.orc_unit_export(self._h, sh, _ptr(kq), _ptr(ks), _ptr(kz), _ptr(vq),
                                  _ptr(vs), _ptr(vz))
        return dict(qtok=qtok, kq=kq, ks=ks, kz=kz, vq=vq, vs=vs, vz=vz)

    def serialize(self, src=None):
        """(bytes u8[R], valid u8[R]) of the unit in the canonical layout
        (``src``: a residual unit's reference)."""
        nbytes = region_bytes(self.kind, self.D, self.cap)
        out = np.zeros(nbytes, np.uint8)
        valid = np.zeros(nbytes, np.uint8)
        rc = self._lib.orc_unit_serialize(self._h, None if src is None else src._h, _ptr(out),
                                          _ptr(valid), nbytes)
        if rc != 0:
            raise ValueError("oracle serialize rejected its input")
        return out, valid


@dataclasses.dataclass
class DecodeResult:
    out: np.ndarray      # fp64 [D]
    lse: float           # natural log
    mask: np.ndarray     # uint32 words over the 4-bit positions
    nsel: int
    weights: np.ndarray  # fp64 softmax weight per attended position


def _override_words(sel_override, npos):
    """Selection override as uint32 words covering npos positions (or None)."""
    if sel_override is None:
        return None
    words = np.zeros(max(npos // G + 2, 1), np.uint32)
    given = np.ascontiguousarray(sel_override, dtype=np.uint32).reshape(-1)
    words[: min(given.size, words.size)] = given[: words.size]
    return words


def decode(unit, q_bits, tau, src=None, sm_scale=0.0, band=1e-6, sel_override=None):
    """Decode one unit for the query ``q_bits`` (bf16 bits [D]).

    ``src`` is the final loop's unit of the same layer, sequence and head when
    ``unit`` is a SHARE unit or a residual (RES2) unit.  ``sel_override``
    (mask words): the selection of positions whose weight is within ``band``
    of ``tau`` (see ``orc_decode_group``).
    """
    D = unit.D
    q = np.ascontiguousarray(q_bits, dtype=np.uint16).reshape(D)
    npos = unit.n
    out = np.zeros(D, np.float64)
    # room beyond npos: a planted mistake in a test copy may write more
    weights = np.zeros(npos + 2, np.float64)
    lse = np.zeros(1, np.float64)
    mask = np.zeros(max(npos // G + 2, 1), np.uint32)
    nw = np.zeros(1, np.int32)
    nsel = np.zeros(1, np.int32)
    ov = _override_words(sel_override, npos)
    rc = unit._lib.orc_decode(unit._h, None if src is None else src._h, _ptr(q),
                         float(tau), float(sm_scale), float(band), _ptr(out),
                         _ptr(lse), _ptr(mask), _ptr(nw), _ptr(nsel),
                         _ptr(ov), _ptr(weights))
    if rc != 0:
        raise ValueError("oracle decode rejected its input")
    return DecodeResult(out=out, lse=float(lse[0]), mask=mask[: nw[0]].copy(),
                        nsel=int(nsel[0]), weights=weights[:npos])


@dataclasses.dataclass
class GroupDecodeResult:
    out: np.ndarray      # fp64 [g][D]
    lse: np.ndarray      # fp64 [g], natural log
    mask: np.ndarray     # uint32 words over the 4-bit positions (union over heads)
    nsel: int
    weights: np.ndarray  # fp64 [g][npos]


def decode_group(unit, q_bits, tau, src=None, sm_scale=0.0, band=1e-6, sel_override=None):
    """Decode one unit for a group of query heads sharing its keys and values.

    ``q_bits``: bf16 bits [g][D].  The selection is the union over the heads;
    ``sel_override`` as in ``decode``.
    """
    D = unit.D
    q = np.ascontiguousarray(q_bits, dtype=np.uint16).reshape(-1, D)
    g = q.shape[0]
    npos = unit.n
    out = np.zeros((g, D), np.float64)
    weights = np.zeros(g * (npos + 2), np.float64)  # room as in decode()
    lse = np.zeros(g, np.float64)
    mask = np.zeros(max(npos // G + 2, 1), np.uint32)
    nw = np.zeros(1, np.int32)
    nsel = np.zeros(1, np.int32)
    ov = _override_words(sel_override, npos)
    rc = unit._lib.orc_decode_group(unit._h, None if src is None else src._h, _ptr(q), g,
                                    float(tau), float(sm_scale), float(band), _ptr(out),
                                    _ptr(lse), _ptr(mask), _ptr(nw), _ptr(nsel),
                                    _ptr(ov), _ptr(weights))
    if rc != 0:
        raise ValueError("oracle decode rejected its input")
    return GroupDecodeResult(out=out, lse=lse, mask=mask[: nw[0]].copy(), nsel=int(nsel[0]),
                             weights=weights[: g * npos].reshape(g, npos).copy())


def plan_brute(n_loops, n_layers, damage, damage_budget, storage_budget_q, sel_milli):
    """Best plan by exhaustive search (cells <= 16): (kinds, reads, damage, storage)
    in the oracle's units, or None when nothing fits the budgets."""
    dmg = np.ascontiguousarray(damage, dtype=np.int32).reshape(-1, 3)
    kinds = np.zeros(n_loops * n_layers, np.uint8)
    r = np.zeros(1, np.int64)
    d = np.zeros(1, np.int64)
    s = np.zeros(1, np.int64)
    rc = _load().orc_plan_brute(n_loops, n_layers, _ptr(dmg), int(damage_budget),
                                int(storage_budget_q), int(sel_milli), _ptr(kinds), _ptr(r),
                                _ptr(d), _ptr(s))
    if rc != 0:
        return None
    return kinds, int(r[0]), int(d[0]), int(s[0])


def vq_decode(idx_k, idx_v, cb_k, cb_v, q_bits, loop, n_loops, sm_scale=0.0):
    """LoopVQ decode of one unit for one loop: idx_k / idx_v u8 [n, D/c],
    cb_k / cb_v fp32 [256, n_loops * c], q bf16 bits [D] -> (out fp64 [D], lse)."""
    idx_k = np.ascontiguousarray(idx_k, dtype=np.uint8)
    idx_v = np.ascontiguousarray(idx_v, dtype=np.uint8)
    cb_k = np.ascontiguousarray(cb_k, dtype=np.float32)
    cb_v = np.ascontiguousarray(cb_v, dtype=np.float32)
    q = np.ascontiguousarray(q_bits, dtype=np.uint16).reshape(-1)
    n, groups = idx_k.shape
    D = q.size
    c = D // groups
    assert idx_v.shape == idx_k.shape and cb_k.shape == (256, n_loops * c) == cb_v.shape
    out = np.zeros(D, np.float64)
    lse = np.zeros(1, np.float64)
    rc = _load().orc_vq_decode(n_loops, D, c, n, int(loop), _ptr(idx_k), _ptr(idx_v), _ptr(cb_k),
                               _ptr(cb_v), _ptr(q), float(sm_scale), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle vq decode rejected its input")
    return out, float(lse[0])


def vq_encode(x_bits, cb, c=4):
    """Codebook indices of one token: x_bits bf16 bits [n_loops, D] (the
    token in every loop of its layer), cb fp32 [256, n_loops * c] -> u8 [D/c]."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    L, D = x.shape
    cb = np.ascontiguousarray(cb, dtype=np.float32)
    assert cb.shape == (256, L * c)
    out = np.zeros(D // c, np.uint8)
    rc = _load().orc_vq_encode(L, D, c, _ptr(x), _ptr(cb), _ptr(out))
    if rc != 0:
        raise ValueError("oracle vq encode rejected its input")
    return out
