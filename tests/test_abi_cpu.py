"""The C-ABI library without a GPU: it builds, loads, exports every function
include/loopkv.h declares, and validates plans on the host.  No CUDA call is
made here (plan_query, status strings and argument checks are host-only)."""

import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "loopkv.h")


@pytest.fixture(scope="module")
def lk():
    from loop_aware_quantized_b200 import build
    build.build()
    from loop_aware_quantized_b200 import loopkv
    return loopkv


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:loopkv_status|void|const char\*)\s+(loopkv_\w+)\s*\(",
                                 text, re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("loopkv_plan_query", "loopkv_plan_load", "loopkv_plan_free",
                     "loopkv_append", "loopkv_decode", "loopkv_set_lengths",
                     "loopkv_check", "loopkv_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lk):
    lib = ctypes.CDLL(lk.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lk):
    for code in range(7):
        assert lk.loopkv_status_string(code)
    assert lk.loopkv_status_string(99) == "unknown status"


def _query(lk, **kw):
    base = dict(n_loops=2, n_layers=2, n_kv_heads=2, head_dim=64, capacity=[64, 96],
                kinds=[0, 2, 1, 0], tau=0.01)
    base.update(kw)
    d, keep = lk.make_desc(base["n_loops"], base["n_layers"], base["n_kv_heads"],
                           base["head_dim"], base["capacity"], base["kinds"], base["tau"])
    rc, sizes = lk.loopkv_plan_query(d)
    return rc, sizes


def test_plan_query_rejects_invalid_plans(lk):
    assert _query(lk)[0] == 0
    assert _query(lk, kinds=[0, 0, 2, 0])[0] == 2          # SHARE in the final loop
    assert _query(lk, n_loops=1, n_layers=4, kinds=[0, 2, 0, 0])[0] == 2
    assert _query(lk, kinds=[0, 5, 1, 0])[0] == 2          # unknown kind
    assert _query(lk, kinds=[0, 0, 4, 0])[0] == 2          # RES2 in the final loop
    assert _query(lk, kinds=[0, 4, 1, 0])[0] == 0          # RES2 in a non-final loop
    assert _query(lk, kinds=[4, 4, 3, 1])[0] == 0          # bf16 and 2-bit references
    assert _query(lk, head_dim=96)[0] == 2
    assert _query(lk, tau=-1.0)[0] == 2
    assert _query(lk, tau=float("nan"))[0] == 2
    assert _query(lk, capacity=[-1, 3])[0] == 2
    assert _query(lk, capacity=[1 << 21, 3])[0] == 2
    assert _query(lk, capacity=list(range(300)))[0] == 2   # max_batch > 256
    rc, _ = lk.loopkv_plan_query(None)
    assert rc == 1


def test_plan_query_checks_the_query_group(lk):
    # query heads per KV head: 1, 2 or 4 (0 reads as 1); the cache does not
    # depend on it (the group shares the KV head's storage)
    base = _query(lk)[1].cache_bytes
    for g in (0, 1, 2, 4):
        d, keep = lk.make_desc(2, 2, 2, 64, [64, 96], [0, 2, 1, 0], 0.01, q_per_kv=g)
        rc, sizes = lk.loopkv_plan_query(d)
        assert rc == 0 and sizes.cache_bytes == base, g
    for g in (-1, 3, 5, 8):
        d, keep = lk.make_desc(2, 2, 2, 64, [64, 96], [0, 2, 1, 0], 0.01, q_per_kv=g)
        assert lk.loopkv_plan_query(d)[0] == 2, g


def test_plan_query_checks_the_decode_split(lk):
    # CTAs per decoded unit: 0 (the library chooses), 1, 2, 4 or 8
    for sp in (0, 1, 2, 4, 8):
        d, keep = lk.make_desc(2, 2, 2, 64, [64, 96], [0, 2, 1, 0], 0.01, decode_split=sp)
        assert lk.loopkv_plan_query(d)[0] == 0, sp
    for sp in (-1, 3, 6, 16):
        d, keep = lk.make_desc(2, 2, 2, 64, [64, 96], [0, 2, 1, 0], 0.01, decode_split=sp)
        assert lk.loopkv_plan_query(d)[0] == 2, sp


def test_binding_loads_only_the_in_tree_library():
    # no environment variable can point the binding at another build
    import subprocess
    import sys
    env = dict(os.environ, LOOPKV_LIBRARY="/nonexistent/libloopkv.so")
    code = ("import sys; sys.path.insert(0, %r); from loop_aware_quantized_b200 import loopkv; "
            "print(loopkv.LIB_PATH)" % ROOT)
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                         check=True).stdout.strip()
    assert out == os.path.join(ROOT, "loop_aware_quantized_b200", "libloopkv.so")


def test_plan_load_checks_arguments_before_any_device_work(lk):
    d, keep = lk.make_desc(2, 2, 2, 64, [64, 96], [0, 2, 1, 0], 0.01)
    rc, h = lk.loopkv_plan_load(d, None, 0, None, 0, None)
    assert rc == 1 and not h.value
    rc, h = lk.loopkv_plan_load(d, ctypes.c_void_p(16), 1, None, 0, None)  # table too small
    assert rc == 1
    rc, h = lk.loopkv_plan_load(d, ctypes.c_void_p(4096), 1 << 20, ctypes.c_void_p(4096 + 8),
                                1 << 30, None)                           # cache misaligned
    assert rc == 1


def test_calls_on_a_null_plan_fail_cleanly(lk):
    cells = np.zeros(1, np.int32)
    n_new = np.ones(1, np.int32)
    p = lk._np_ptr
    assert lk.loopkv_append(None, p(cells), 1, 1, p(n_new), 1, None, None, None) == 1
    assert lk.loopkv_decode(None, p(cells), 1, 1, None, None, None, None, 0, None, None) == 1
    assert lk.loopkv_set_lengths(None, p(cells), 1, 1, p(n_new), None) == 1
    assert lk.loopkv_check(None, None) == 1
    assert lk.loopkv_unit_region(None, 0, 0, 0)[0] == 1
    lk.loopkv_plan_free(None)


def test_cache_size_matches_the_oracle_layout(lk):
    """Two independent implementations of the canonical layout agree on every
    unit's region size (library plan_query vs oracle region_bytes)."""
    from oracle import oracle as orc
    from synth import workloads as W
    for config in ("0", "1", "2", "2r", "4"):
        wl = W.make(config)
        rc, sizes = _query(lk, n_loops=wl.n_loops, n_layers=wl.n_layers, n_kv_heads=wl.n_heads,
                           head_dim=wl.head_dim, capacity=wl.capacity, kinds=wl.kinds,
                           tau=wl.tau)
        assert rc == 0
        total = 0
        for c in range(wl.n_cells):
            for b in range(wl.batch):
                total += wl.n_heads * orc.region_bytes(int(wl.kinds[c]), wl.head_dim,
                                                       int(wl.capacity[b]))
        assert total == sizes.cache_bytes, config


def test_config2_cache_fits_one_b200(lk):
    from synth import workloads as W
    wl = W.make("2")
    rc, sizes = _query(lk, n_loops=4, n_layers=24, n_kv_heads=16, head_dim=128,
                       capacity=wl.capacity, kinds=wl.kinds, tau=wl.tau)
    assert rc == 0 and sizes.cache_bytes < 120e9


def test_vq_decode_checks_arguments_before_any_device_work(lk):
    # every host check of the LoopVQ decode runs before a CUDA call, so it
    # answers without a GPU
    import ctypes
    import numpy as np
    assert lk.loopkv_vq_decode(None, 0, None, None, None, None, None, None, None, None, None) == 1
    d = lk.loopkv_vq_desc(4, 2, 2, 128, 3, 704, 0.0)
    lens = np.array([1, 33, 700], np.int32)
    lp = lens.ctypes.data_as(ctypes.c_void_p)
    fake = ctypes.c_void_p(1 << 20)   # aligned, never dereferenced on these paths
    args = [fake] * 6
    assert lk.loopkv_vq_decode(d, 0, lp, None, *args[1:], None, None) == 1   # null index array
    assert lk.loopkv_vq_decode(d, 4, lp, *args, None, None) == 1             # loop out of range
    bad = np.array([1, 0, 3], np.int32)
    assert lk.loopkv_vq_decode(d, 0, bad.ctypes.data_as(ctypes.c_void_p), *args, None, None) == 1
    odd = ctypes.c_void_p((1 << 20) + 4)
    assert lk.loopkv_vq_decode(d, 0, lp, odd, *args[1:], None, None) == 1    # misaligned
    d.head_dim = 96
    assert lk.loopkv_vq_decode(d, 0, lp, *args, None, None) == 1


def test_vq_encode_checks_arguments_before_any_device_work(lk):
    import ctypes
    import numpy as np
    d = lk.loopkv_vq_desc(4, 2, 2, 128, 2, 16, 0.0)
    pos = np.array([3, 0], np.int32)
    pp = pos.ctypes.data_as(ctypes.c_void_p)
    fake = ctypes.c_void_p(1 << 20)   # aligned, never dereferenced on these paths
    assert lk.loopkv_vq_encode(None, pp, 5, fake, fake, fake, None) == 1
    assert lk.loopkv_vq_encode(d, pp, 0, None, None, None, None) == 0      # nothing to do
    assert lk.loopkv_vq_encode(d, pp, -1, fake, fake, fake, None) == 1
    assert lk.loopkv_vq_encode(d, pp, 14, fake, fake, fake, None) == 1     # 3 + 14 > 16
    assert lk.loopkv_vq_encode(d, pp, 5, None, fake, fake, None) == 1
    assert lk.loopkv_vq_encode(d, pp, 5, fake, ctypes.c_void_p((1 << 20) + 8), fake, None) == 1


def test_header_is_plain_c(tmp_path):
    # the boundary is a C ABI: the header compiles as ISO C99 with no C++ or
    # CUDA types, and every declared function is extern "C" for C++ callers
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "use.c"
    src.write_text('#include "loopkv.h"\nint main(void) { return sizeof(loopkv_vq_desc) == 0; }\n')
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                           "-I", os.path.join(root, "include"), "-c", str(src),
                           "-o", str(tmp_path / "use.o")])


def test_binding_checks_tensors_before_passing_pointers(lk):
    # the library sees only pointers: the binding refuses host tensors, wrong
    # dtypes, layouts and shapes itself, with LOOPKV_ERR_INVALID_ARG and no
    # call into the library (these inputs never reach a device)
    import torch
    where = "test"
    host = torch.zeros((2, 3, 4), dtype=torch.float32)
    with pytest.raises(lk.LoopKVError) as e:
        lk._need(host, where, "out", (torch.float32,))
    assert e.value.status == 1 and "CUDA" in str(e.value)
    with pytest.raises(lk.LoopKVError) as e:
        lk._need(np.zeros(3), where, "out", (torch.float32,))
    assert e.value.status == 1 and "torch tensor" in str(e.value)
    with pytest.raises(lk.LoopKVError):
        lk._need(None, where, "q", (torch.bfloat16,))
    lk._need(None, where, "lse", (torch.float32,), optional=True)
    with pytest.raises(lk.LoopKVError) as e:
        lk._host_ints([1, 2, 3], where, "lengths", 2)
    assert "2 values" in str(e.value)
    assert list(lk._host_ints((4, 5), where, "lengths", 2)) == [4, 5]
    # the public LoopVQ calls run the same checks first
    ik = torch.zeros((2, 3, 2, 16, 32), dtype=torch.uint8)
    cb = torch.zeros((2, 2, 256, 16), dtype=torch.float32)
    q = torch.zeros((2, 3, 2, 128), dtype=torch.bfloat16)
    with pytest.raises(lk.LoopKVError) as e:
        lk.vq_decode(0, np.array([1, 1, 1]), ik, ik, cb, cb, q)
    assert e.value.status == 1
    x = torch.zeros((4, 2, 3, 2, 1, 128), dtype=torch.bfloat16)
    with pytest.raises(lk.LoopKVError) as e:
        lk.vq_encode(np.zeros(3, np.int32), x, cb, ik)
    assert e.value.status == 1
    with pytest.raises(lk.LoopKVError):
        lk.plan_optimize(2, 2, 64, np.zeros((3, 3)), 1, 1000)   # damage for 3 of 4 cells
