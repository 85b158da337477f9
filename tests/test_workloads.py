"""The seeded input generators (CPU only): deterministic, and with the structure their recipes state."""
import torch

from paged_kv_cache_tree_b200 import workloads as wl


def test_verify_workload_is_deterministic_and_well_formed():
    a = wl.make_workload("tiny")
    b = wl.make_workload("tiny")
    for f in ("q", "k_cache", "v_cache", "k_new", "v_new"):
        assert torch.equal(getattr(a, f).view(torch.int16), getattr(b, f).view(torch.int16))
    assert torch.equal(a.block_tables, b.block_tables)
    # every mapped physical block is used by exactly one sequence
    mapped = a.block_tables[a.block_tables >= 0]
    assert mapped.unique().numel() == mapped.numel()
    # candidates sit at P_b + i
    for bb in range(a.B):
        n, L = int(a.num_candidates[bb]), int(a.context_lens[bb])
        assert a.slot_offsets[bb, :n].tolist() == list(range(L - n, L))


def test_e4m3_caches_are_nan_exactly_where_the_16_bit_caches_are():
    w = wl.make_workload("tiny")
    c8 = wl.make_e4m3_cache(w)
    for src, codes in ((w.k_cache, c8.k_cache), (w.v_cache, c8.v_cache)):
        nan_code = (codes & 0x7F) == 0x7F
        assert torch.equal(nan_code, torch.isnan(src))
    assert torch.equal(c8.k_cache, wl.make_e4m3_cache(w).k_cache)
    assert ((c8.k_scale >= 0.004) & (c8.k_scale <= 0.012)).all()


def test_prefix_inputs_tables_and_starts():
    pi = wl.make_prefix_inputs(n_cached=30, n_prompts=10, stem_len=(0, 50), tail_len=(0, 100), prompt_tail=(0, 40))
    assert torch.equal(pi.cached_tokens, wl.make_prefix_inputs(n_cached=30, n_prompts=10, stem_len=(0, 50),
                                                               tail_len=(0, 100), prompt_tail=(0, 40)).cached_tokens)
    st = pi.cached_starts
    assert (st[1:] >= st[:-1]).all() and int(st[-1]) == pi.cached_tokens.numel()
    used = pi.cached_tables[pi.cached_tables >= 0]
    assert used.unique().numel() == used.numel() and int(used.max()) < pi.num_blocks
    for i, s in enumerate(pi.seqs("cached")):
        assert int((pi.cached_tables[i] >= 0).sum()) == (len(s) + pi.bs - 1) // pi.bs


def test_lookahead_inputs_separators_and_ranges():
    li = wl.make_lookahead_inputs(B=8, hist_len=(0, 200), n_docs=3, doc_len=(10, 100), vocab=50, copy_len=(2, 5))
    assert (li.history >= 0).all()
    assert int((li.global_tokens < 0).sum()) == 3           # one separator after each document
    assert ((li.copy_len >= 2) & (li.copy_len <= 5)).all()
    assert [len(h) for h in li.histories()] == (li.hist_starts[1:] - li.hist_starts[:-1]).tolist()
