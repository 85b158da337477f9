"""Pins of the acceptance oracle (oracle/tree_accept.py) against closed forms, a brute force over all
root-to-node paths, an independent mask construction and a pure-Python argmax scan."""
import math

import numpy as np
import pytest
import torch

from oracle import tree_accept as ta
from paged_kv_cache_tree_b200 import workloads as wl


def random_forest(rng, C):
    return [int(rng.integers(-1, i)) if i > 0 else -1 for i in range(C)]


# ------------------------------------------------------------------------------------------ masks
def test_chain_masks_closed_form():
    C = 12
    parents = np.array([[i - 1 for i in range(C)]])
    m = ta.tree_masks(parents, np.array([C]))
    assert [int(x) for x in m[0]] == [(1 << (i + 1)) - 1 for i in range(C)]


def test_masks_match_the_input_generators_construction():
    rng = np.random.default_rng(1)
    for _ in range(50):
        C = int(rng.integers(1, 33))
        n = int(rng.integers(0, C + 1))
        par = random_forest(rng, C)
        got = ta.tree_masks(np.array([par]), np.array([n]))[0]
        want = wl.masks_from_parents(par, n)
        assert [int(x) for x in got] == want


def test_mask_rows_past_n_are_zero_and_roots_see_only_themselves():
    par = np.array([[-1, -1, 0, 2, -1]])
    m = ta.tree_masks(par, np.array([4]))[0]
    assert [int(x) for x in m] == [0b1, 0b10, 0b101, 0b1101, 0]


# ------------------------------------------------------------------------------------------ argmax
def scan_argmax(row):
    best, bi = -math.inf, 0
    for i, v in enumerate(row):
        v = -math.inf if math.isnan(v) else v
        if v > best:
            best, bi = v, i
    return bi


def test_argmax_equals_a_scalar_scan_with_ties_and_nans():
    rng = np.random.default_rng(2)
    x = rng.integers(-3, 4, size=(40, 37)).astype(np.float64)   # many ties
    x[3, :] = np.nan
    x[5, [0, 7, 9]] = np.nan
    x[6, :] = -np.inf
    got = ta.logits_argmax(x)
    assert list(got) == [scan_argmax(r) for r in x]
    assert got[3] == 0 and got[6] == 0


def test_argmax_finds_the_planted_margin():
    w = wl.make_workload("tiny")
    a = wl.make_accept_inputs(w, vocab=5000)
    x = ta.logits_argmax(__import__("oracle").widen_to_f64(wl.to_numpy_bits(a.target_logits), w.dtype).reshape(-1, 5000))
    assert np.array_equal(x.reshape(a.planted.shape), a.planted.numpy())


# ------------------------------------------------------------------------------------------ acceptance
def run(tokens, parents, amax, n, L):
    return ta.greedy_accept(np.array([amax]), np.array([tokens]), np.array([parents]), np.array([n]), np.array([L]))


def test_chain_all_correct_accepts_everything():
    C, L = 6, 50
    parents = [i - 1 for i in range(C)]
    amax = [10 + r for r in range(C + 1)]           # row r predicts token 10 + r
    tokens = [10 + i for i in range(C)]             # candidate i follows row i (its parent's row)
    acc, path, bonus, slots = run(tokens, parents, amax, C, L)
    assert acc[0] == C
    assert list(path[0]) == list(range(C))
    assert bonus[0] == 10 + C
    assert list(slots[0]) == [L - C + i for i in range(C)]


@pytest.mark.parametrize("k", [0, 1, 3, 5])
def test_chain_first_miss_stops_the_path(k):
    C, L = 6, 40
    parents = [i - 1 for i in range(C)]
    amax = [10 + r for r in range(C + 1)]
    tokens = [10 + i for i in range(C)]
    tokens[k] = 999
    acc, path, bonus, slots = run(tokens, parents, amax, C, L)
    assert acc[0] == k
    assert list(path[0][:k]) == list(range(k)) and all(x == -1 for x in path[0][k:])
    assert bonus[0] == amax[k]                       # row of the last accepted node (row 0 if none)
    assert all(s == -1 for s in slots[0][k:])


def test_star_accepts_the_smallest_correct_root():
    parents = [-1] * 5
    amax = [7] + [0] * 5
    tokens = [3, 7, 4, 7, 7]
    acc, path, bonus, slots = run(tokens, parents, amax, 5, 20)
    assert acc[0] == 1 and path[0][0] == 1 and bonus[0] == amax[2]
    assert list(slots[0]) == [-1, 15, -1, -1, -1]


def test_candidates_past_n_are_ignored():
    parents = [-1, 0, 1, 2]
    amax = [1, 2, 3, 4, 5]
    tokens = [1, 2, 3, 4]
    acc, path, bonus, slots = run(tokens, parents, amax, 2, 30)
    assert acc[0] == 2 and bonus[0] == 3 and list(slots[0]) == [28, 29, -1, -1]


def brute_force(tokens, parents, amax, n):
    """All root-to-node paths by DFS over child lists; the deepest fully correct one, smallest node."""
    children = {i: [] for i in range(-1, n)}
    for i in range(n):
        children[parents[i]].append(i)
    best = (0, -1, [])

    def dfs(node, row, path):
        nonlocal best
        for c in children[node]:
            if tokens[c] != amax[row]:
                continue
            p2 = path + [c]
            if len(p2) > best[0] or (len(p2) == best[0] and c < best[1]):
                best = (len(p2), c, p2)
            dfs(c, c + 1, p2)

    dfs(-1, 0, [])
    return best


def test_acceptance_matches_a_brute_force_over_all_paths():
    rng = np.random.default_rng(3)
    for _ in range(300):
        C = int(rng.integers(1, 17))
        n = int(rng.integers(0, C + 1))
        parents = random_forest(rng, C)
        amax = [int(x) for x in rng.integers(0, 3, C + 1)]     # a 3-token vocabulary: many hits
        tokens = [int(x) for x in rng.integers(0, 3, C)]
        L = n + int(rng.integers(0, 20))
        acc, path, bonus, slots = run(tokens, parents, amax, n, L)
        depth, node, bpath = brute_force(tokens, parents, amax, n)
        assert acc[0] == depth
        assert [int(x) for x in path[0][:depth]] == bpath
        assert bonus[0] == amax[0 if node < 0 else node + 1]
        for d, j in enumerate(bpath):
            assert slots[0][j] == L - n + d
            assert d == 0 or parents[j] == bpath[d - 1]
        assert sum(1 for s in slots[0] if s >= 0) == depth


def test_generated_inputs_give_partial_acceptance():
    w = wl.make_workload("tree", fill="zero")
    w = wl.make_workload(dict(wl.WORKLOADS["tree"], B=4, ctx=("fixed", [100, 200, 300, 400])), fill="zero")
    a = wl.make_accept_inputs(w, vocab=3000)
    amax = a.planted.numpy()
    acc, path, bonus, slots = ta.greedy_accept(amax, a.tokens.numpy(), w.parents.numpy(), w.num_candidates.numpy(),
                                               w.context_lens.numpy())
    assert 0 <= acc.min() and acc.max() <= w.C
    assert acc.sum() > 0
