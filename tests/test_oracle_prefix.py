"""Pins of the prefix-tree oracle (CPU only): a brute force over the inserted sequences, closed forms
and counts that do not go through the trie."""
import random

import pytest

from oracle.prefix_cache import PrefixTree, batch_insert_choices, insert_batch, lookup_batch


def brute_match(prompt, inserted, bs):
    """Longest run of leading full blocks of ``prompt`` that some inserted sequence shares, and the
    block of each matched prefix taken from the first sequence (in insertion order) that has it."""
    best = 0
    for s, _ in inserted:
        k = 0
        while (k + 1) * bs <= min(len(prompt), len(s)) and list(prompt[:(k + 1) * bs]) == list(s[:(k + 1) * bs]):
            k += 1
        best = max(best, k)
    blocks = []
    for j in range(best):
        pre = list(prompt[:(j + 1) * bs])
        for s, t in inserted:
            if len(s) >= (j + 1) * bs and list(s[:(j + 1) * bs]) == pre:
                blocks.append(int(t[j]))
                break
    return best, blocks


def corpus(rng, n, bs, vocab=5, max_len=90):
    """Small-vocabulary sequences built from a few shared stems, so that prefixes collide often."""
    stems = [[rng.randrange(vocab) for _ in range(rng.randrange(0, 40))] for _ in range(4)]
    seqs = []
    for _ in range(n):
        s = list(rng.choice(stems)) + [rng.randrange(vocab) for _ in range(rng.randrange(0, max_len - 40))]
        seqs.append(s)
    return seqs


@pytest.mark.parametrize("bs", [1, 2, 4, 16])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_lookup_equals_brute_force(bs, seed):
    rng = random.Random(seed * 10 + bs)
    seqs = corpus(rng, 30, bs)
    next_block = [100]

    def table(s):
        t = list(range(next_block[0], next_block[0] + len(s) // bs + 1))
        next_block[0] += len(t)
        return t

    inserted = [(s, table(s)) for s in seqs]
    tree = PrefixTree(bs)
    insert_batch(tree, [s for s, _ in inserted], [t for _, t in inserted])
    prompts = corpus(rng, 40, bs) + [s[: rng.randrange(len(s) + 1)] for s in seqs[:10]]
    for p in prompts:
        m, blocks = brute_match(p, inserted, bs)
        assert tree.lookup(p) == blocks
        assert len(blocks) == m


def test_a_sequence_finds_all_its_full_blocks_and_partial_blocks_never_count():
    bs = 4
    tree = PrefixTree(bs)
    s = list(range(10))                     # 2 full blocks + 2 tokens
    assert tree.insert(s, [7, 8, 9]) == [7, 8]
    assert tree.lookup(s) == [7, 8]
    assert tree.lookup(s[:7]) == [7]        # the second block is incomplete
    assert tree.lookup(s[:3]) == []
    assert tree.lookup([]) == []
    assert tree.lookup(s + [99, 98]) == [7, 8]   # 3rd block (8, 9, 99, 98) is not cached
    assert tree.count == 2


def test_first_inserter_owns_a_prefix_and_later_ones_reuse_it():
    bs = 2
    tree = PrefixTree(bs)
    a, b = [1, 2, 3, 4], [1, 2, 5, 6]
    assert tree.insert(a, [10, 11]) == [10, 11]
    assert tree.insert(b, [20, 21]) == [10, 21]   # block (1, 2) is shared; (5, 6) under it is new
    assert tree.insert(a, [30, 31]) == [10, 11]   # nothing new
    assert tree.lookup([1, 2, 5, 6, 7]) == [10, 21]
    assert tree.count == 3


def test_same_block_tokens_under_different_parents_are_different_nodes():
    bs = 2
    tree = PrefixTree(bs)
    tree.insert([1, 1, 9, 9], [1, 2])
    tree.insert([2, 2, 9, 9], [3, 4])
    assert tree.lookup([2, 2, 9, 9]) == [3, 4]
    assert tree.lookup([9, 9]) == []
    assert tree.count == 4


@pytest.mark.parametrize("seed", [3, 4])
def test_node_count_is_the_number_of_distinct_block_prefixes(seed):
    rng = random.Random(seed)
    bs = 3
    seqs = corpus(rng, 50, bs, vocab=3)
    tree = PrefixTree(bs)
    insert_batch(tree, seqs, [list(range(1000 * i, 1000 * i + 40)) for i in range(len(seqs))])
    distinct = {tuple(s[:(j + 1) * bs]) for s in seqs for j in range(len(s) // bs)}
    assert tree.count == len(distinct)


def test_batch_choices_contain_the_sequential_result_and_pin_existing_nodes():
    rng = random.Random(9)
    bs = 2
    before = PrefixTree(bs)
    old = corpus(rng, 10, bs, vocab=3)
    insert_batch(before, old, [list(range(500 + 50 * i, 550 + 50 * i)) for i in range(len(old))])
    batch = corpus(rng, 20, bs, vocab=3)
    tables = [list(range(5000 + 50 * i, 5050 + 50 * i)) for i in range(len(batch))]
    choices = batch_insert_choices(before, batch, tables)
    seq_tree = PrefixTree(bs)
    insert_batch(seq_tree, old, [list(range(500 + 50 * i, 550 + 50 * i)) for i in range(len(old))])
    got = insert_batch(seq_tree, batch, tables)
    for row_c, row_g, s in zip(choices, got, batch):
        assert len(row_c) == len(s) // bs
        for j, (c, g) in enumerate(zip(row_c, row_g)):
            assert g in c
            if j < len(before.lookup(s)):
                assert c == {g}
    assert lookup_batch(seq_tree, batch) == got
