"""GPU parity of the prefix-tree KV lookup and insert against the CPU oracle (needs a B200).

Every output is an integer (block ids, match lengths), so comparisons are exact. Inserts of one
sequence per call follow the oracle's sequential semantics block for block; a batch inserted in one call
may give a new prefix to any of the sequences that add it, so there the unique parts (match lengths,
existing nodes) are compared exactly and the rest is checked for validity and consistency.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_tree_b200 as taco
from oracle.prefix_cache import PrefixTree, batch_insert_choices, insert_batch, lookup_batch
from paged_kv_cache_tree_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def starts_of(seqs):
    return torch.tensor([0] + list(np.cumsum([len(s) for s in seqs])), dtype=torch.int32)


def flat(seqs):
    return torch.tensor([t for s in seqs for t in s], dtype=torch.int32)


def padded(rows, width):
    out = np.full((len(rows), width), -1, dtype=np.int32)
    for i, r in enumerate(rows):
        out[i, :len(r)] = r
    return out


def small_inputs(seed, bs=16, n_cached=40, n_prompts=48, vocab=50):
    return wl.make_prefix_inputs(n_cached=n_cached, n_prompts=n_prompts, bs=bs, n_stems=4, stem_len=(0, 120),
                                 tail_len=(0, 300), prompt_tail=(0, 100), vocab=vocab, seed=seed)


def gpu_cache(pi, capacity=None):
    cap = capacity or 1 << int(np.ceil(np.log2(max(4, 2 * pi.num_blocks))))
    return taco.PrefixCache(pi.num_blocks, pi.bs, cap)


@pytest.mark.parametrize("bs", [1, 16, 64])
def test_sequential_inserts_and_lookups_are_bit_exact(bs):
    pi = small_inputs(seed=bs, bs=bs, n_cached=24, vocab=4)
    cached, tables = pi.seqs("cached"), pi.cached_tables.numpy()
    cache = gpu_cache(pi)
    tree = PrefixTree(bs)
    for i, s in enumerate(cached):          # one sequence per call: the oracle's order
        got, cnt = cache.insert(flat([s]).cuda(), starts_of([s]).cuda(), torch.from_numpy(tables[i:i + 1]).cuda())
        want = tree.insert(s, tables[i])
        assert taco.check_device() == 0
        assert got.cpu().numpy()[0].tolist() == want + [-1] * (pi.max_blocks - len(want))
        assert int(cnt[0]) == len(want)
    prompts = pi.seqs("prompts") + [s[: len(s) // 2] for s in cached[:8]] + [[], [1] * (bs - 1 if bs > 1 else 0)]
    blocks, matched = cache.lookup(flat(prompts).cuda(), starts_of(prompts).cuda(), pi.max_blocks)
    assert taco.check_device() == 0
    want = lookup_batch(tree, prompts)
    assert matched.cpu().tolist() == [len(w) for w in want]
    assert np.array_equal(blocks.cpu().numpy(), padded(want, pi.max_blocks))
    # the node arrays hold exactly the oracle's nodes
    depth = cache.node_depth.cpu().numpy()
    assert int((depth >= 0).sum()) == tree.count


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_one_call_batch_insert_is_valid_and_lookups_agree(seed):
    pi = small_inputs(seed=10 + seed, vocab=3)
    cached, tables = pi.seqs("cached"), pi.cached_tables.numpy()
    cache = gpu_cache(pi)
    got, cnt = cache.insert(pi.cached_tokens.cuda(), pi.cached_starts.cuda(), pi.cached_tables.cuda())
    assert taco.check_device() == 0
    got = got.cpu().numpy()
    choices = batch_insert_choices(PrefixTree(pi.bs), cached, tables)
    owner = {}
    for i, s in enumerate(cached):
        nfull = len(s) // pi.bs
        assert int(cnt[i]) == nfull
        assert (got[i, nfull:] == -1).all()
        for j in range(nfull):
            assert int(got[i, j]) in choices[i][j]
            key = tuple(s[:(j + 1) * pi.bs])
            assert owner.setdefault(key, int(got[i, j])) == int(got[i, j]), "one prefix, two nodes"
    tree = PrefixTree(pi.bs)
    insert_batch(tree, cached, tables)
    assert int((cache.node_depth.cpu().numpy() >= 0).sum()) == tree.count == len(owner)
    prompts = pi.seqs("prompts")
    blocks, matched = cache.lookup(pi.prompts.cuda(), pi.prompt_starts.cuda(), pi.max_blocks)
    assert taco.check_device() == 0
    want_len = [len(w) for w in lookup_batch(tree, prompts)]
    assert matched.cpu().tolist() == want_len
    blocks = blocks.cpu().numpy()
    for i, p in enumerate(prompts):
        want = [owner[tuple(p[:(j + 1) * pi.bs])] for j in range(want_len[i])]
        assert blocks[i].tolist() == want + [-1] * (pi.max_blocks - len(want))


def test_second_batch_reuses_existing_nodes_exactly():
    pi = small_inputs(seed=7, vocab=3, n_cached=30)
    cached, tables = pi.seqs("cached"), pi.cached_tables.numpy()
    first, second = cached[:15], cached[15:]
    cache = gpu_cache(pi)
    before = PrefixTree(pi.bs)
    for i, s in enumerate(first):
        cache.insert(flat([s]).cuda(), starts_of([s]).cuda(), torch.from_numpy(tables[i:i + 1]).cuda())
        before.insert(s, tables[i])
    got, _ = cache.insert(flat(second).cuda(), starts_of(second).cuda(), torch.from_numpy(tables[15:]).cuda())
    assert taco.check_device() == 0
    choices = batch_insert_choices(before, second, tables[15:])
    got = got.cpu().numpy()
    n_pinned = 0
    for i, s in enumerate(second):
        pre = before.lookup(s)
        for j in range(len(s) // pi.bs):
            assert int(got[i, j]) in choices[i][j]
            if j < len(pre):
                assert int(got[i, j]) == pre[j]
                n_pinned += 1
    assert n_pinned > 0


def test_full_size_cache_and_prompts():
    """The bench's prefix workload: 256 cached sequences (about 0.9 M tokens, 34 k nodes) inserted one
    per call in order, then all 64 prompts looked up in one call, bit-exact against the oracle."""
    pi = wl.make_prefix_inputs()
    cached, tables = pi.seqs("cached"), pi.cached_tables
    cache = gpu_cache(pi)
    tok, st = pi.cached_tokens.cuda(), pi.cached_starts
    for i in range(len(cached)):
        s0, s1 = int(st[i]), int(st[i + 1])
        cache.insert(tok[s0:s1], torch.tensor([0, s1 - s0], dtype=torch.int32).cuda(), tables[i:i + 1].cuda())
    assert taco.check_device() == 0
    tree = PrefixTree(pi.bs)
    insert_batch(tree, cached, tables.tolist())
    blocks, matched = cache.lookup(pi.prompts.cuda(), pi.prompt_starts.cuda(), pi.max_blocks)
    assert taco.check_device() == 0
    want = lookup_batch(tree, pi.seqs("prompts"))
    assert matched.cpu().tolist() == [len(w) for w in want]
    assert np.array_equal(blocks.cpu().numpy(), padded(want, pi.max_blocks))


def test_max_blocks_caps_the_walk_and_partial_blocks_never_match():
    bs = 4
    s = list(range(30))
    cache = taco.PrefixCache(16, bs, 64)
    table = torch.arange(8, dtype=torch.int32).view(1, 8).cuda()
    got, cnt = cache.insert(flat([s]).cuda(), starts_of([s]).cuda(), table[:, :3])   # only 3 blocks fit
    assert got.cpu().tolist() == [[0, 1, 2]] and int(cnt[0]) == 3
    prompts = [s, s[:11], s[:3]]
    blocks, matched = cache.lookup(flat(prompts).cuda(), starts_of(prompts).cuda(), 5)
    assert matched.cpu().tolist() == [3, 2, 0]
    assert blocks.cpu().tolist() == [[0, 1, 2, -1, -1], [0, 1, -1, -1, -1], [-1] * 5]
    assert taco.check_device() == 0


def test_device_errors_are_reported_not_faulted():
    bs = 2
    cache = taco.PrefixCache(8, bs, 4)                      # 4 slots
    s = list(range(20))                                     # 10 blocks: more nodes than slots
    table = torch.arange(10, dtype=torch.int32).view(1, 10) % 8
    got, cnt = cache.insert(flat([s]).cuda(), starts_of([s]).cuda(), table.cuda())
    with pytest.raises(taco.TacoError) as ei:
        taco.check_device()
    assert "table full" in str(ei.value)
    # the blocks claim slots together, so which of them got the 4 slots is not fixed; the walk ends at
    # the first block without one, and every block before it is inserted with its own block id
    n = int(cnt[0])
    assert 0 <= n <= 4
    assert got.cpu().tolist()[0] == table[0, :n].tolist() + [-1] * (10 - n)
    # a block id outside the pool, and decreasing seq_starts
    cache = taco.PrefixCache(8, bs, 64)
    bad = torch.tensor([[0, 99, 2]], dtype=torch.int32).cuda()
    got, cnt = cache.insert(flat([s[:6]]).cuda(), starts_of([s[:6]]).cuda(), bad)
    with pytest.raises(taco.TacoError) as ei:
        taco.check_device()
    assert "block id" in str(ei.value)
    assert got.cpu().tolist() == [[0, -1, -1]] and int(cnt[0]) == 1
    blocks, matched = cache.lookup(flat([s]).cuda(), torch.tensor([4, 2], dtype=torch.int32).cuda(), 4)
    with pytest.raises(taco.TacoError):
        taco.check_device()
    assert matched.cpu().tolist() == [0]
    assert taco.check_device() == 0


def test_insert_wait_for_an_unpublished_slot_times_out_and_reports_it():
    """A slot holding a block's key whose node was never published (a claim by a writer that never
    finished) makes the inserting warp wait; the wait is bounded, so the call returns, reports
    TACO_DEVERR_WAIT_TIMEOUT, inserts nothing past that block, and the next clean call is exact.
    Nothing else runs in the kernel (no copy is in flight), so running out of the wait faults nothing."""
    bs = 4
    s = [7, 1, 7, 2, 5, 5, 3, 3]                             # two full blocks
    tree = PrefixTree(bs)
    cache = taco.PrefixCache(16, bs, 64)
    got, cnt = cache.insert(flat([s]).cuda(), starts_of([s]).cuda(), torch.tensor([[3, 9]], dtype=torch.int32).cuda())
    assert taco.check_device() == 0
    assert got.cpu().tolist()[0][:2] == tree.insert(s, [3, 9]) == [3, 9]
    # un-publish the first block's node: its slot keeps the key, its node index goes back to -1
    keys, nodes = cache.slot_keys.cpu(), cache.slot_nodes.cpu()
    first = [i for i in range(cache.capacity) if int(keys[i]) != 0 and int(nodes[i]) == 3]
    assert len(first) == 1
    cache.slot_nodes[first[0]] = -1
    got, cnt = cache.insert(flat([s]).cuda(), starts_of([s]).cuda(), torch.tensor([[5, 6]], dtype=torch.int32).cuda())
    with pytest.raises(taco.TacoError) as ei:
        taco.check_device()
    assert "wait timed out" in str(ei.value)
    assert int(cnt[0]) == 0 and got.cpu().tolist() == [[-1, -1]]
    assert taco.check_device() == 0                          # the word was cleared by the read above
    # a clean cache afterwards behaves exactly like the oracle
    cache = taco.PrefixCache(16, bs, 64)
    tree = PrefixTree(bs)
    for table in ([3, 9], [5, 6]):
        got, cnt = cache.insert(flat([s]).cuda(), starts_of([s]).cuda(), torch.tensor([table], dtype=torch.int32).cuda())
        assert taco.check_device() == 0
        want = tree.insert(s, table)
        assert got.cpu().tolist()[0][:len(want)] == want and int(cnt[0]) == len(want)
