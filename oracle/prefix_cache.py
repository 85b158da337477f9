"""CPU oracle for the prefix-tree KV lookup used to skip prefill work.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module. The product path never calls it, and this module imports
nothing from the product.

What the pages say (618zxw.cn page, section "プレフィックスキャッシュ技術を使用してTTFTを削減する";
the 17173xz.com overview's prefill paragraph; the tencentcloud.com document's list of techniques, which
names automatic prefix caching): the KV caches of earlier requests' prefill are kept in a prefix-tree
structure (on GPU and CPU), so that prefill turns into a lookup of cached KV, and only the tokens that
are not found go through prefill compute. The pages fix no granularity, key or interface. The
readings taken here:

* The tree's nodes are full KV blocks of ``bs`` tokens. A node is identified by the whole token prefix
  it ends (its own ``bs`` tokens under its parent's path); the first block of a sequence hangs from
  the root. A partial trailing block is never cached or matched.
* A node owns the physical KV block that holds its tokens' K/V.
* ``lookup(prompt)`` returns the longest run of leading full blocks of the prompt whose path exists in
  the tree, as the physical blocks along that path (a block-table prefix); the matched token count is
  that many blocks times ``bs``.
* ``insert(tokens, blocks)`` adds the full blocks of a sequence whose K/V sit in ``blocks`` (its
  block table): a block whose prefix is already in the tree keeps the existing node, otherwise the
  sequence's own block becomes the node. It returns, per full block, the physical block that holds
  that prefix afterwards. A batch is inserted sequence by sequence in index order.

Pinned by tests against a brute force over the inserted sequences (longest common full-block prefix,
first inserter of each prefix), closed forms (a sequence finds all of its own full blocks, partial
blocks never count) and the count of distinct block prefixes.
"""
from __future__ import annotations


class PrefixTree:
    """A trie whose edges are tuples of ``bs`` token ids; each node holds a physical block id."""

    def __init__(self, bs: int):
        if bs < 1:
            raise ValueError("bs must be >= 1")
        self.bs = int(bs)
        self.children = {}   # root's children: block tokens (tuple) -> node
        self.count = 0

    def _blocks(self, tokens):
        toks = [int(t) for t in tokens]
        return [tuple(toks[j * self.bs:(j + 1) * self.bs]) for j in range(len(toks) // self.bs)]

    def lookup(self, tokens) -> list:
        """Physical blocks of the longest cached run of leading full blocks of ``tokens``."""
        path = []
        level = self.children
        for blk in self._blocks(tokens):
            node = level.get(blk)
            if node is None:
                break
            path.append(node["block"])
            level = node["children"]
        return path

    def insert(self, tokens, blocks) -> list:
        """Insert the full blocks of one sequence whose j-th block is ``blocks[j]``; returns, per full
        block, the block that holds that prefix afterwards."""
        out = []
        level = self.children
        for j, blk in enumerate(self._blocks(tokens)):
            node = level.get(blk)
            if node is None:
                node = {"block": int(blocks[j]), "children": {}}
                level[blk] = node
                self.count += 1
            out.append(node["block"])
            level = node["children"]
        return out


def insert_batch(tree: PrefixTree, seqs, tables) -> list:
    """Sequential batch insertion (sequence 0 first); returns one list of blocks per sequence."""
    return [tree.insert(s, t) for s, t in zip(seqs, tables)]


def lookup_batch(tree: PrefixTree, prompts) -> list:
    return [tree.lookup(p) for p in prompts]


def batch_insert_choices(tree_before: PrefixTree, seqs, tables) -> list:
    """For a batch inserted concurrently, where the order among the batch is not fixed: per sequence
    and full block, the set of physical blocks that may hold that prefix afterwards (the existing
    node's block if the prefix was cached before the batch, else the own block of any batch sequence
    that has the same prefix)."""
    bs = tree_before.bs
    owners = {}
    for s, t in zip(seqs, tables):
        toks = tuple(int(x) for x in s)
        for j in range(len(toks) // bs):
            owners.setdefault(toks[:(j + 1) * bs], set()).add(int(t[j]))
    out = []
    for s in seqs:
        before = tree_before.lookup(s)
        toks = tuple(int(x) for x in s)
        row = []
        for j in range(len(toks) // bs):
            row.append({before[j]} if j < len(before) else owners[toks[:(j + 1) * bs]])
        out.append(row)
    return out
