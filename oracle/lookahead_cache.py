"""CPU oracle for the batched Lookahead Cache: candidate forests from earlier occurrences of a sequence's
most recent tokens.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module. The product path never calls it, and this module imports nothing
from the product.

What the pages say (53ai.com workshop page, "整体方案分为两大部分", item 1 "基于批处理的 Lookahead Cache",
and the paragraphs after it): candidates for a whole batch are predicted at once; what is generated next
has often appeared before, in the prompt or in earlier output, so when the most recent tokens match an
earlier passage the tokens that followed it are proposed; each sequence keeps a local cache and the
batch shares a global one; the cache is queried by match length and proposes a preset amount of copied
tokens (copy_len), which is penalised adaptively from the batch size and each request's hit rate;
the proposals form a forest (several branches) to raise the hit rate. The learned weighting of tree
shapes is left out. The readings taken here:

* The local cache of sequence b is its own history h_b (prompt plus generated tokens); the global cache
  is one shared token array g. A token value below 0 in g separates passages and never matches.
* Match: for each cache separately, the longest m in [1, min(M, n_b)] such that the last m tokens of
  h_b occur in that cache ending at a position e with a following token (e < length; for the local
  cache e < n_b, i.e. an earlier occurrence). Occurrences of that m are taken most recent first
  (larger e first).
* A continuation is the cache's tokens from e on, at most copy_len_b of them, stopping before a
  separator or the end.
* The forest is a trie of at most C candidate nodes: the local continuations in order, then the global
  ones, each inserted as a path from the current position (a path's leading tokens already in the
  trie are shared); nodes are numbered in creation order, so a parent always precedes its children;
  insertion stops when C nodes exist (a path is cut at the budget).
* copy_len update after a verify step: hit_b <- (1 - a) hit_b + a * accepted_b / max(1, proposed_b),
  copy_len_b = clamp(floor(copy_max * hit_b * min(1, B_ref / B) + 0.5), 1, copy_max), in float32 in
  this order (the same precision on the GPU decides the same integer).

Pinned by tests against a brute force over all windows, closed forms on periodic sequences and a
hand-worked example.
"""
from __future__ import annotations

import numpy as np


def longest_match(context, cache, max_match: int, local: bool):
    """(m, ends): the longest m whose last-m-token key occurs in ``cache`` with a following token, and
    the end positions e of those occurrences, most recent first. For the local cache the key's own
    position is excluded because it has no following token there. (0, []) when nothing matches."""
    n = len(context)
    limit = len(cache)
    best_m, best = 0, []
    for m in range(1, min(max_match, n) + 1):
        key = list(context[n - m:])
        ends = []
        for e in range(m, limit):           # occurrence cache[e - m : e], following token cache[e]
            if local and e >= n:
                break
            window = list(cache[e - m:e])
            if window == key and int(cache[e]) >= 0 and all(int(t) >= 0 for t in window):
                ends.append(e)
        if ends:
            best_m, best = m, sorted(ends, reverse=True)
    return best_m, best


def continuation(cache, e: int, copy_len: int):
    out = []
    for t in cache[e:e + copy_len]:
        if int(t) < 0:
            break
        out.append(int(t))
    return out


def build_forest(paths, C: int):
    """Insert token paths into a trie of at most C nodes; returns (tokens, parents) in creation order."""
    tokens, parents = [], []
    children = {}                           # (parent, token) -> node
    for path in paths:
        parent = -1
        for t in path:
            node = children.get((parent, t))
            if node is None:
                if len(tokens) >= C:
                    return tokens, parents
                node = len(tokens)
                tokens.append(t)
                parents.append(parent)
                children[(parent, t)] = node
            parent = node
    return tokens, parents


def propose(history, global_cache, max_match: int, copy_len: int, C: int):
    """Candidate forest of one sequence: (tokens, parents, m_local, m_global)."""
    m_l, ends_l = longest_match(history, history, max_match, local=True)
    m_g, ends_g = longest_match(history, global_cache, max_match, local=False)
    paths = [continuation(history, e, copy_len) for e in ends_l]
    paths += [continuation(global_cache, e, copy_len) for e in ends_g]
    tokens, parents = build_forest([p for p in paths if p], C)
    return tokens, parents, m_l, m_g


def propose_batch(histories, global_cache, max_match: int, copy_len, C: int):
    """Per sequence: padded arrays tokens, parents [B, C] (-1 past n_b) and n_b."""
    B = len(histories)
    tok = np.full((B, C), -1, dtype=np.int32)
    par = np.full((B, C), -1, dtype=np.int32)
    n = np.zeros(B, dtype=np.int32)
    for b, h in enumerate(histories):
        t, p, _, _ = propose(h, global_cache, max_match, int(copy_len[b]), C)
        tok[b, :len(t)] = t
        par[b, :len(p)] = p
        n[b] = len(t)
    return tok, par, n


def update_copy_len(hit, accepted, proposed, batch: int, copy_max: int, alpha: float, batch_ref: int):
    """The copy_len rule above, in float32. Returns (new hit [B] float32, copy_len [B] int32)."""
    f = np.float32
    hit = np.asarray(hit, dtype=f)
    rate = np.asarray(accepted, dtype=f) / np.maximum(np.asarray(proposed, dtype=f), f(1))
    new_hit = (f(1) - f(alpha)) * hit + f(alpha) * rate
    scale = f(min(1.0, float(f(batch_ref) / f(batch))))
    x = f(copy_max) * new_hit * scale + f(0.5)
    cl = np.clip(np.floor(x).astype(np.int64), 1, copy_max).astype(np.int32)
    return new_hit.astype(f), cl
