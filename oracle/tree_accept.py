"""CPU oracle for the step after the verify: tree masks, greedy acceptance, KV compaction plan.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module. The product path never calls it, and this module imports
nothing from the product.

What the pages say ("大模型倍速推理引擎 TACO-LLM 的设计与实践", 53ai.com workshop page, sections
"TACO-LLM 如何解决大模型推理瓶颈?", "优化方案设计思路", "整体方案分为两大部分" and "优化策略总结"):
the target model validates, in one forward pass, candidate tokens obtained ahead of time, and so
emits several tokens per step; the candidates are organised as a forest (multi-branch prediction),
and what matters is the hit length of the candidates. The pages fix no acceptance rule. The reading
taken here is the plain greedy one:

* Candidate i of sequence b (i < n_b) carries token ``tokens[b][i]`` and parent ``parents[b][i]``
  (-1 for a root, else an earlier candidate). Row 0 of the target's logits is its prediction after
  the committed prefix, row i + 1 its prediction after candidate i.
* Candidate i is correct iff its token equals the target's argmax in the row of its parent (row 0
  for a root). The argmax is the smallest index among the maximal values; NaN counts as -inf; a row
  with no number in it gives index 0.
* A candidate is accepted iff it and all its ancestors are correct. The hit is the deepest accepted
  candidate (ties: the smallest index); the accepted path runs from its root down to it, and its
  length is the hit length (0 when nothing is accepted).
* The target's argmax after the last accepted node (row 0 when nothing is accepted) is one more
  token the step emits (the bonus token).
* The accepted candidates' K/V move to the contiguous tail: the candidate at depth d (1-based) of
  the path goes to logical slot P_b + d - 1 (P_b = L_b - n_b); everything else gets -1. These slot
  offsets are the input of a paged KV-append with the step's k_new / v_new.
* The tree mask word of candidate i has bit j set iff j is i or an ancestor of i.

Every function here is pinned by tests (closed forms on chains and stars, invariants of the path, a
brute force over all root-to-node paths, ``numpy.argmax`` and a pure-Python scan for the argmax).
"""
from __future__ import annotations

import numpy as np


def ancestors(parents_row, i: int) -> list:
    """Candidate i and its ancestors, from i up to its root, by walking parent links."""
    out = []
    j = i
    while j >= 0:
        out.append(j)
        j = int(parents_row[j])
    return out


def tree_masks(parents: np.ndarray, num_candidates: np.ndarray) -> np.ndarray:
    """uint32 [B, C]: bit j of word (b, i) is set iff j is i or an ancestor of i (rows i >= n_b: 0)."""
    parents = np.asarray(parents)
    B, C = parents.shape
    out = np.zeros((B, C), dtype=np.uint32)
    for b in range(B):
        for i in range(int(num_candidates[b])):
            word = 0
            for j in ancestors(parents[b], i):
                word |= 1 << j
            out[b, i] = word
    return out


def logits_argmax(logits: np.ndarray) -> np.ndarray:
    """int32 [rows]: per row the smallest index of the largest value (NaN as -inf; all-NaN -> 0).

    ``logits`` is float64 [rows, V] (widen 16-bit patterns with ``widen_to_f64`` first).
    """
    x = np.where(np.isnan(logits), -np.inf, logits)
    return np.argmax(x, axis=1).astype(np.int32)


def greedy_accept(target_argmax: np.ndarray, tokens: np.ndarray, parents: np.ndarray,
                  num_candidates: np.ndarray, context_lens: np.ndarray):
    """Greedy acceptance of a candidate forest.

    target_argmax int [B, C + 1]; tokens, parents int [B, C]; num_candidates, context_lens int [B].
    Returns (accept_len [B], path [B, C] (-1 padded), bonus [B], slot_offsets [B, C] (-1 = skip)).
    """
    target_argmax = np.asarray(target_argmax)
    B, C = np.asarray(tokens).shape
    accept_len = np.zeros(B, dtype=np.int32)
    path = np.full((B, C), -1, dtype=np.int32)
    bonus = np.zeros(B, dtype=np.int32)
    slots = np.full((B, C), -1, dtype=np.int32)
    for b in range(B):
        n = int(num_candidates[b])
        correct = []
        for i in range(n):
            p = int(parents[b, i])
            row = 0 if p < 0 else p + 1
            correct.append(int(tokens[b, i]) == int(target_argmax[b, row]))
        best, best_depth = -1, 0
        for i in range(n):
            chain = ancestors(parents[b], i)
            if all(correct[j] for j in chain) and len(chain) > best_depth:
                best, best_depth = i, len(chain)
        accept_len[b] = best_depth
        if best >= 0:
            chain = ancestors(parents[b], best)[::-1]  # root first
            P = int(context_lens[b]) - n
            for d, j in enumerate(chain):
                path[b, d] = j
                slots[b, j] = P + d
        bonus[b] = int(target_argmax[b, 0 if best < 0 else best + 1])
    return accept_len, path, bonus, slots
