"""Pins of the oracle's routing steps (top-k, counts, offsets, slot rows, permute).

Each check compares the oracle against something other than itself: brute
force enumeration, direct counting definitions, invariants, or the
hand-derived fixture under tests/golden/.
"""

import itertools
import json
import os

import numpy as np
import pytest

from oracle import moe_ref as ref


def _brute_topk(l, k):
    """Best k-subset by logit sum; ties -> lexicographically smallest index set;
    then ordered by (-l, e)."""
    E = len(l)
    best, best_set = None, None
    for comb in itertools.combinations(range(E), k):  # lexicographic order
        s = sum(l[c] for c in comb)
        if best is None or s > best:
            best, best_set = s, comb
    return sorted(best_set, key=lambda e: (-l[e], e))


@pytest.mark.parametrize("E,k", [(5, 1), (5, 2), (5, 3), (6, 6), (7, 4)])
def test_topk_matches_brute_force_with_ties(E, k):
    rng = np.random.default_rng(E * 10 + k)
    l = rng.integers(-2, 3, size=(300, E)).astype(np.float64)  # many ties
    idx = ref.topk_select(l, k)
    for t in range(l.shape[0]):
        assert list(idx[t]) == _brute_topk(list(l[t]), k)


def test_topk_signed_zero_and_extremes_tie_lowest_index():
    l = np.array([[0.0, -0.0, -1.0, 0.0], [-1e300, 1e300, 1e300, -0.5]])
    assert ref.topk_select(l, 2).tolist() == [[0, 1], [1, 2]]


def _brute_slots(idx):
    T, k = idx.shape
    slot = np.zeros_like(idx)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            before = sum(1 for tt in range(T) for jj in range(k) if idx[tt, jj] < e)
            same = sum(1 for tt in range(t) if e in idx[tt])
            slot[t, j] = before + same
    return slot


@pytest.mark.parametrize("T,E,k", [(17, 5, 2), (9, 4, 4), (23, 8, 3)])
def test_counts_offsets_slots_against_counting_definition(T, E, k):
    rng = np.random.default_rng(T + E + k)
    l = rng.normal(size=(T, E))
    if E > 4:
        l[:, E - 1] -= 50.0  # force an empty expert
    r = ref.route_from_logits(l, k)
    idx = r["idx"]
    for t in range(T):
        assert len(set(idx[t])) == k
    assert r["counts"].sum() == T * k
    assert r["offsets"][0] == 0 and r["offsets"][-1] == T * k
    for e in range(E):
        assert r["counts"][e] == int(np.sum(idx == e))
        assert r["offsets"][e + 1] - r["offsets"][e] == r["counts"][e]
    assert np.array_equal(r["slot_row"], _brute_slots(idx))
    # perm is a bijection onto [0, T*k)
    assert sorted(r["slot_row"].ravel().tolist()) == list(range(T * k))
    src = r["perm_src"]
    for e in range(E):
        seg = src[r["offsets"][e]:r["offsets"][e + 1]]
        assert np.all(np.diff(seg) > 0), "segment rows must be in ascending token order"
        assert all(e in idx[t] for t in seg)


def test_permute_rows_are_source_tokens():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(11, 6))
    r = ref.route_from_logits(rng.normal(size=(11, 5)), 3)
    xp = ref.permute(x, r["slot_row"])
    assert np.array_equal(xp, x[r["perm_src"]])


def test_top_k_equals_E_every_expert_gets_every_token():
    T, E = 13, 4
    r = ref.route_from_logits(np.random.default_rng(0).normal(size=(T, E)), E)
    assert np.all(r["counts"] == T)
    assert np.array_equal(r["slot_row"], r["idx"] * T + np.arange(T)[:, None])


def test_golden_routing_fixture(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "routing_tiny.json")))
    r = ref.route_from_logits(np.array(fx["logits"], dtype=np.float64), fx["top_k"])
    for key in ("idx", "counts", "offsets", "slot_row", "perm_src"):
        assert r[key].tolist() == fx[key], key
    np.testing.assert_allclose(r["gate"], np.array(fx["gate"]), rtol=1e-15)


def test_softmax_is_shift_invariant_and_normalised():
    rng = np.random.default_rng(5)
    l = rng.normal(size=(7, 9)) * 30
    p = ref.softmax(l)
    np.testing.assert_allclose(p.sum(1), 1.0, rtol=1e-15)
    np.testing.assert_allclose(ref.softmax(l + 123.0), p, rtol=1e-13)
    # a two-expert softmax is the logistic function of the logit difference
    l2 = rng.normal(size=(50, 2))
    np.testing.assert_allclose(ref.softmax(l2)[:, 0],
                               1.0 / (1.0 + np.exp(l2[:, 1] - l2[:, 0])), rtol=1e-14)


def test_select_logits_drive_discrete_steps_only():
    rng = np.random.default_rng(9)
    l = rng.normal(size=(8, 6))
    sel = l.copy()
    sel[:, 0] += 100.0  # the device decided differently
    r = ref.route_from_logits(l, 2, select_logits=sel)
    assert np.all(r["idx"][:, 0] == 0)
    np.testing.assert_allclose(r["gate"][:, 0], ref.softmax(l)[:, 0])


# ---- routing_stats: closed forms of special cases ---------------------------

def test_routing_stats_uniform_and_one_hot():
    st = ref.routing_stats([5, 5, 5, 5], C=5)
    assert list(st) == [20, 5, 1, 1, 0, 0, 0, 1]
    st = ref.routing_stats([12, 0, 0, 0], C=4)          # everything on one expert
    assert np.allclose(st, [12, 3, 4, 0, np.sqrt(3), 3, 8 / 12, 4 / 16], rtol=1e-15, atol=0)
    assert list(ref.routing_stats([0, 0, 0])) == [0, 0, 0, 0, 0, 3, 0, 0]


def test_routing_stats_two_values():
    # half the experts hold a rows, half b rows: cv = |a - b| / (a + b)
    a, b, E = 7, 1, 6
    st = ref.routing_stats([a, b] * (E // 2), C=3)
    mean = (a + b) / 2
    assert np.isclose(st[4], abs(a - b) / (a + b))
    assert np.isclose(st[2], a / mean) and np.isclose(st[3], b / mean)
    assert np.isclose(st[6], (E // 2) * (a - 3) / ((a + b) * E // 2))


def test_routing_stats_of_a_real_routing_matches_its_padded_layout():
    rng = np.random.default_rng(3)
    T, E, k = 200, 8, 2
    l = rng.normal(size=(T, E)) + np.linspace(0, 3, E)      # skewed
    r = ref.route_from_logits(l, k)
    C = ref.capacity(T * k, E)
    st = ref.routing_stats(r["counts"], C)
    pad = ref.padded_layout(r["idx"], r["slot_row"], r["offsets"], C)
    assert np.isclose(st[6], np.mean(pad < 0))                # dropped pairs
    assert np.isclose(st[7], np.sum(pad >= 0) / (E * C))      # used slots
