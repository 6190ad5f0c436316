"""Pins for the oracle's routing: numpy's stable argsort (library routine),
histogram invariants, the review thread's structured case and a hand-derived
golden fixture."""
import os

import numpy as np
import pytest

import oracle
from workloads import structured_routing

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("T,k,E,seed", [(100, 3, 8, 0), (1, 1, 1, 1), (257, 6, 384, 2), (64, 8, 256, 3)])
def test_route_matches_stable_argsort(T, k, E, seed):
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, E, (T, k)).astype(np.int64)
    r = oracle.route(idx, E)
    flat = idx.ravel()
    assert np.array_equal(r["count"], np.bincount(flat, minlength=E))
    assert r["count"].sum() == T * k
    assert np.array_equal(r["offset"], np.concatenate([[0], np.cumsum(r["count"])]))
    assert np.array_equal(r["perm"], np.argsort(flat, kind="stable"))
    assert np.array_equal(r["inv"][r["perm"]], np.arange(T * k))
    assert r["dropped"] == 0


def test_route_structured_case_is_uniform():
    idx, _ = structured_routing(96, 4, 12)
    r = oracle.route(idx.numpy(), 12)
    assert np.all(r["count"] == 96 * 4 // 12)


def test_route_drops_out_of_range_ids():
    idx = np.array([[0, 5], [-1, 1], [2, 2]], np.int64)
    r = oracle.route(idx, 3)
    assert r["dropped"] == 2
    assert list(r["count"]) == [1, 1, 2]
    assert list(r["perm"]) == [0, 3, 4, 5]
    assert list(r["inv"]) == [0, -1, -1, 1, 2, 3]


def test_route_golden_fixture():
    """tests/golden/routing_T4_k2_E3.txt: a 4-token, top-2, 3-expert case
    with a duplicated expert, derived by hand from the stable-sort reading."""
    vals = {}
    with open(os.path.join(GOLDEN, "routing_T4_k2_E3.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                key, rest = line.split(":")
                vals[key.strip()] = [int(v) for v in rest.split()]
    idx = np.array(vals["topk_idx"], np.int64).reshape(4, 2)
    r = oracle.route(idx, 3)
    for key in ("count", "offset", "perm", "inv"):
        assert list(r[key]) == vals[key], key
