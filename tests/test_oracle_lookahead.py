"""Pins of the Lookahead Cache oracle (CPU only): a window-index brute force, closed forms on periodic
sequences, hand-worked examples and forest invariants."""
import random

import numpy as np
import pytest

from oracle.lookahead_cache import build_forest, longest_match, propose, propose_batch, update_copy_len


def brute_longest(context, cache, M, local):
    """Index every window of every length once (a dict of tuples), then read the answer off it."""
    n, N = len(context), len(cache)
    index = {}
    for m in range(1, M + 1):
        for e in range(m, N):
            w = tuple(int(x) for x in cache[e - m:e])
            if min(w) < 0 or int(cache[e]) < 0 or (local and e >= n):
                continue
            index.setdefault(w, []).append(e)
    for m in range(min(M, n), 0, -1):
        ends = index.get(tuple(int(x) for x in context[n - m:]), [])
        if ends:
            return m, sorted(ends, reverse=True)
    return 0, []


@pytest.mark.parametrize("seed", range(6))
def test_longest_match_equals_window_index(seed):
    rng = random.Random(seed)
    for _ in range(40):
        h = [rng.randrange(3) for _ in range(rng.randrange(0, 60))]
        g = [rng.choice([0, 1, 2, -1]) for _ in range(rng.randrange(0, 80))]
        M = rng.randrange(1, 6)
        assert longest_match(h, h, M, True) == brute_longest(h, h, M, True)
        assert longest_match(h, g, M, False) == brute_longest(h, g, M, False)


def test_hand_worked_example():
    # key (5, 6) ends at 2 (next 7) and at 5 (next 8); the most recent one comes first
    h = [5, 6, 7, 5, 6, 8, 5, 6]
    assert longest_match(h, h, 2, True) == (2, [5, 2])
    assert longest_match(h, h, 4, True) == (2, [5, 2])     # (8, 5, 6) and longer never occurred before
    tok, par, m_l, m_g = propose(h, [], 4, 3, 6)
    assert (tok, par, m_l, m_g) == ([8, 5, 6, 7, 5, 6], [-1, 0, 1, -1, 3, 4], 2, 0)
    tok, par, _, _ = propose(h, [], 4, 3, 4)               # the budget cuts the second path
    assert (tok, par) == ([8, 5, 6, 7], [-1, 0, 1, -1])


def test_periodic_history_gives_one_chain():
    h = [1, 2, 3] * 10
    for copy_len in (1, 2, 3, 7):
        tok, par, m_l, _ = propose(h, [], 4, copy_len, 32)
        assert m_l == 4
        assert tok == [(1, 2, 3)[i % 3] for i in range(copy_len)]  # every occurrence continues the cycle
        assert par == list(range(-1, copy_len - 1))


def test_global_cache_separators_stop_matches_and_continuations():
    h = [9, 4, 4]
    g = [7, 4, 4, 1, 2, -1, 4, 4, 3, -1, 4]
    m, ends = longest_match(h, g, 3, False)
    assert (m, ends) == (2, [8, 3])          # (4, 4) at 1..3 -> 1 and at 6..8 -> 3; the last 4 has no next
    tok, par, m_l, m_g = propose(h, g, 3, 5, 8)
    assert (m_l, m_g) == (1, 2)             # local: (4,) ends at 2 with next 4
    assert tok == [4, 3, 1, 2] and par == [-1, -1, -1, 2]
    # local continuation [4] from e=2; global [3] (stops at -1) then [1, 2] (stops at -1)


def test_empty_and_unmatched():
    assert propose([], [1, 2], 3, 4, 8)[:2] == ([], [])
    assert propose([5], [1, 2, 3], 3, 4, 8)[:2] == ([], [])


@pytest.mark.parametrize("seed", range(4))
def test_forest_invariants(seed):
    rng = random.Random(100 + seed)
    for _ in range(30):
        paths = [[rng.randrange(3) for _ in range(rng.randrange(0, 6))] for _ in range(rng.randrange(0, 10))]
        C = rng.randrange(1, 33)
        tok, par = build_forest(paths, C)
        assert len(tok) == len(par) <= C
        assert all(-1 <= p < i for i, p in enumerate(par))
        seen = set()
        for i, p in enumerate(par):          # siblings carry distinct tokens
            assert (p, tok[i]) not in seen
            seen.add((p, tok[i]))
        # every node is a prefix of some path
        def path_of(i):
            out = []
            while i >= 0:
                out.append(tok[i])
                i = par[i]
            return out[::-1]
        for i in range(len(tok)):
            q = path_of(i)
            assert any(p[:len(q)] == q for p in paths)
        if sum(len(p) for p in paths) <= C:   # with room for everything, every path is present
            for p in paths:
                for k in range(1, len(p) + 1):
                    assert any(path_of(i) == p[:k] for i in range(len(tok)))


def test_batch_padding():
    hs = [[1, 2, 1, 2], [3], [1, 1, 1]]
    tok, par, n = propose_batch(hs, [], 2, np.array([2, 2, 5]), 4)
    assert n.tolist() == [2, 0, 1]
    assert tok[0].tolist() == [1, 2, -1, -1] and par[0].tolist() == [-1, 0, -1, -1]
    assert tok[1].tolist() == [-1] * 4 and tok[2].tolist() == [1, -1, -1, -1]


def test_copy_len_update_hand_values():
    hit, cl = update_copy_len([0.5, 0.0, 1.0, 0.25], [4, 0, 0, 8], [8, 0, 5, 8], batch=8, copy_max=8,
                              alpha=0.5, batch_ref=16)
    # rates 0.5, 0 (0/1), 0, 1 -> hits 0.5, 0, 0.5, 0.625 -> copy 4.5->4, 0.5->1 (clamped), 4.5->4, 5.5->5
    assert hit.tolist() == [0.5, 0.0, 0.5, 0.625]
    assert cl.tolist() == [4, 1, 4, 5]
    _, cl = update_copy_len([1.0], [8], [8], batch=64, copy_max=8, alpha=0.5, batch_ref=16)
    assert cl.tolist() == [2]               # 8 * 1 * 16/64 = 2


def test_copy_len_rounds_half_up():
    # rate 7/8 = 0.875, hit 0.5*0.5 + 0.5*0.875 = 0.6875, 8 * 0.6875 = 5.5 -> 6 (round half up)
    hit, cl = update_copy_len([0.5], [7], [8], batch=4, copy_max=8, alpha=0.5, batch_ref=16)
    assert hit.tolist() == [0.6875] and cl.tolist() == [6]
    # 8 * 0.3 = 2.4 -> 2 (in float32 the products stay below 2.5)
    _, cl = update_copy_len([0.3], [3], [10], batch=1, copy_max=8, alpha=0.5, batch_ref=16)
    assert cl.tolist() == [2]
