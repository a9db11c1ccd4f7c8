"""The planner (loopkv_plan_optimize, host code in the library) against the
CPU oracle's exhaustive search, on small random profiles.  No GPU."""

import time

import numpy as np
import pytest

from oracle import oracle as orc


@pytest.fixture(scope="module")
def lk():
    from loop_aware_quantized_b200 import loopkv
    return loopkv


def _cost(kinds, n_loops, n_layers, damage, sel_milli):
    """Reads (thousandths of a quarter of D bytes), damage, storage (quarters)
    of a plan, from the cost readings of the oracle's planner."""
    N = n_layers
    reads = dmg = sto = 0
    for c, k in enumerate(kinds):
        dmg += int(damage[c][k])
        if k == 0:
            reads += 5000 + sel_milli
            sto += 6
        elif k == 1:
            reads += 4000
            sto += 4
        else:
            f = kinds[(n_loops - 1) * N + c % N]
            reads += 5000 + sel_milli if f == 0 else 4000
    return reads, dmg, sto


@pytest.mark.parametrize("n_loops,n_layers", [(1, 3), (2, 2), (2, 4), (3, 3), (4, 2), (4, 3)])
def test_planner_matches_exhaustive_search(lk, n_loops, n_layers):
    rng = np.random.default_rng(100 * n_loops + n_layers)
    cells = n_loops * n_layers
    D = 128
    q = D // 4
    for trial in range(12):
        damage = rng.integers(0, 20, size=(cells, 3))
        damage[:, 0] = rng.integers(0, 4, size=cells)          # 4-bit: least damage
        sel = float(rng.choice([0.0, 0.003, 0.25]))
        sel_milli = int(round(1000 * sel))
        dmax = int(damage.max(axis=1).sum())
        dbud = int(rng.integers(0, dmax + 1))
        sbud_q = int(rng.integers(0, 6 * cells + 1))
        ref = orc.plan_brute(n_loops, n_layers, damage, dbud, sbud_q, sel_milli)
        try:
            kinds, cost = lk.plan_optimize(n_loops, n_layers, D, damage, dbud, sbud_q * q, sel)
        except lk.LoopKVError as e:
            assert ref is None and e.args[0].startswith("loopkv_plan_optimize"), (trial, ref)
            continue
        assert ref is not None, trial
        r, d, s = _cost(kinds, n_loops, n_layers, damage, sel_milli)
        # the unique optimum: fewest reads, then damage, then storage
        assert (r, d, s) == (ref[1], ref[2], ref[3]), (trial, (r, d, s), ref[1:])
        assert d <= dbud and s <= sbud_q
        assert cost["reads"] == pytest.approx(r * q / 1000.0) and cost["damage"] == d
        assert cost["storage"] == s * q
        final = kinds[(n_loops - 1) * n_layers:]
        assert (final != 2).all()                               # no SHARE in the final loop


def test_planner_budget_extremes(lk):
    n_loops, n_layers, D = 2, 3, 64
    damage = np.array([[1, 5, 3], [2, 6, 4], [0, 3, 9], [1, 2, 9], [2, 2, 9], [0, 1, 9]])
    # unlimited: every cell reads as little as it can; SHARE beats a tie in reads on damage
    kinds, cost = lk.plan_optimize(n_loops, n_layers, D, damage, 10 ** 6, 10 ** 6)
    # final loop 2-bit (fewest reads); cells 0, 1 SHARE it (same reads, less
    # damage than their own 2-bit), cell 2 keeps its own 2-bit (SHARE costs 9)
    assert list(kinds) == [2, 2, 1, 1, 1, 1]
    assert cost["reads"] == 6 * D and cost["damage"] == 3 + 4 + 3 + 2 + 2 + 1
    # storage for nothing but the final loop's 2-bit cells forces SHARE elsewhere
    kinds, cost = lk.plan_optimize(n_loops, n_layers, D, damage, 10 ** 6, 3 * D)
    assert list(kinds[:3]) == [2, 2, 2] and list(kinds[3:]) == [1, 1, 1]
    # a zero damage budget needs a zero-damage choice in every cell
    with pytest.raises(lk.LoopKVError):
        lk.plan_optimize(n_loops, n_layers, D, damage, 0, 10 ** 6)
    # more budget never means more reads
    prev = None
    for b in range(0, 40):
        try:
            _, cost = lk.plan_optimize(n_loops, n_layers, D, damage, b, 10 ** 6)
        except lk.LoopKVError:
            continue
        assert prev is None or cost["reads"] <= prev
        prev = cost["reads"]


def test_planner_rejects_bad_arguments(lk):
    import ctypes
    dmg = np.zeros((4, 3), np.int32)
    with pytest.raises(lk.LoopKVError):
        lk.plan_optimize(2, 2, 96, dmg, 1, 1000)                 # head_dim
    with pytest.raises(lk.LoopKVError):
        lk.plan_optimize(7, 1, 64, np.zeros((7, 3)), 1, 1000)    # more than 6 loops
    with pytest.raises(lk.LoopKVError):
        lk.plan_optimize(2, 2, 64, -np.ones((4, 3)), 1, 1000)    # negative damage
    with pytest.raises(lk.LoopKVError):
        lk.plan_optimize(2, 2, 64, dmg, 1, 1000, sel_fraction=1.5)
    rc, _ = lk.loopkv_plan_optimize(None, None)
    assert rc == 1


def test_planner_full_model_shape(lk):
    # 4 loops x 24 layers with a damage budget resolution of ~1000 units
    rng = np.random.default_rng(7)
    n_loops, n_layers, D = 4, 24, 128
    cells = n_loops * n_layers
    damage = np.stack([rng.integers(0, 3, cells), rng.integers(5, 20, cells),
                       rng.integers(2, 30, cells)], axis=1)
    all_q4 = 6 * cells * (D // 4)
    t0 = time.perf_counter()
    kinds, cost = lk.plan_optimize(n_loops, n_layers, D, damage, 1000, int(0.65 * all_q4), 0.002)
    el = time.perf_counter() - t0
    r, d, s = _cost(kinds, n_loops, n_layers, damage, 2)
    assert d <= 1000 and s * (D // 4) <= int(0.65 * all_q4)
    assert cost["reads"] == pytest.approx(r * (D // 4) / 1000.0)
    assert el < 60, el
