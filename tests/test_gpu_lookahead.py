"""GPU parity of the Lookahead Cache (candidate forests and the copy_len update) against the CPU oracle
(needs a B200). Outputs are integers (tokens, parents, counts) and float32 hit rates computed in the
same order on both sides, so every comparison is exact."""
import numpy as np
import pytest
import torch

import paged_kv_cache_tree_b200 as taco
from oracle import lookahead_cache as la
from oracle import tree_accept as ta
from paged_kv_cache_tree_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def run_gpu(li):
    d = li.to("cuda")
    tok, par, num = taco.lookahead_propose(d.history, d.hist_starts, d.global_tokens, d.copy_len, li.max_match, li.C)
    assert taco.check_device() == 0
    return tok.cpu().numpy(), par.cpu().numpy(), num.cpu().numpy()


def check_exact(li):
    tok, par, num = run_gpu(li)
    wt, wp, wn = la.propose_batch(li.histories(), li.global_tokens.tolist(), li.max_match, li.copy_len.numpy(), li.C)
    assert np.array_equal(num, wn)
    assert np.array_equal(tok, wt)
    assert np.array_equal(par, wp)
    return wn


@pytest.mark.parametrize("vocab,p_phrase", [(3, 0.0), (8, 0.5), (1000, 0.9)])
@pytest.mark.parametrize("C,max_match", [(16, 4), (32, 1), (5, 16)])
def test_forests_bit_exact_small(vocab, p_phrase, C, max_match):
    li = wl.make_lookahead_inputs(B=24, hist_len=(0, 300), n_docs=4, doc_len=(0, 400), n_phrases=20, phrase_len=(2, 6),
                                  p_phrase=p_phrase, vocab=vocab, copy_len=(0, 9), max_match=max_match, C=C,
                                  seed=vocab + C)
    n = check_exact(li)
    assert n.max() > 0


def test_many_occurrences_take_the_ordered_fallback():
    """More than 1024 occurrences of the longest match: periodic histories and a periodic global cache."""
    hist = [[1, 2] * 1500, [7, 7, 7] * 600 + [8], [5] * 2000]
    glob = ([1, 2, 3] * 800 + [-1]) * 2
    li = wl.LookaheadInputs(history=torch.tensor(sum(hist, []), dtype=torch.int32),
                            hist_starts=torch.tensor([0, 3000, 4801, 6801], dtype=torch.int32),
                            global_tokens=torch.tensor(glob, dtype=torch.int32),
                            copy_len=torch.tensor([8, 6, 3], dtype=torch.int32), max_match=4, C=32)
    check_exact(li)


def test_empty_histories_no_global_and_copy_len_zero():
    li = wl.LookaheadInputs(history=torch.tensor([1, 2, 1, 2, 1], dtype=torch.int32),
                            hist_starts=torch.tensor([0, 0, 5, 5], dtype=torch.int32),
                            global_tokens=torch.zeros(0, dtype=torch.int32),
                            copy_len=torch.tensor([4, 4, 0], dtype=torch.int32), max_match=3, C=8)
    tok, par, num = run_gpu(li)
    assert num.tolist() == [0, 2, 0]
    assert tok[1, :2].tolist() == [2, 1] and par[1, :2].tolist() == [-1, 0]
    check_exact(li)


def test_full_size_workload_and_forests_feed_the_mask_kernel():
    li = wl.make_lookahead_inputs()
    n = check_exact(li)
    assert (n > 0).mean() > 0.5
    # the proposed forests are valid inputs of the tree-mask step
    tok, par, num = run_gpu(li)
    masks = taco.tree_mask_from_parents(torch.from_numpy(par).cuda(), torch.from_numpy(num).cuda())
    assert taco.check_device() == 0
    assert np.array_equal(masks.cpu().numpy().view(np.uint32), ta.tree_masks(par, num))


def test_copy_len_update_bit_exact():
    rng = np.random.default_rng(3)
    for B in (1, 7, 64, 300):
        hit = rng.random(B).astype(np.float32)
        prop = rng.integers(0, 17, B).astype(np.int32)
        acc = np.minimum(rng.integers(0, 17, B), prop).astype(np.int32)
        h = torch.from_numpy(hit).cuda()
        cl = torch.zeros(B, dtype=torch.int32, device="cuda")
        taco.lookahead_update_copy_len(torch.from_numpy(acc).cuda(), torch.from_numpy(prop).cuda(), h, cl, copy_max=8,
                                       alpha=0.3, batch_ref=16)
        want_hit, want_cl = la.update_copy_len(hit, acc, prop, batch=B, copy_max=8, alpha=0.3, batch_ref=16)
        assert np.array_equal(h.cpu().numpy().view(np.uint32), want_hit.view(np.uint32))
        assert np.array_equal(cl.cpu().numpy(), want_cl)


def test_bad_starts_are_reported_not_faulted():
    li = wl.LookaheadInputs(history=torch.tensor([1, 2, 1, 2], dtype=torch.int32),
                            hist_starts=torch.tensor([3, 1], dtype=torch.int32),
                            global_tokens=torch.zeros(0, dtype=torch.int32),
                            copy_len=torch.tensor([4], dtype=torch.int32), max_match=2, C=8)
    d = li.to("cuda")
    tok, par, num = taco.lookahead_propose(d.history, d.hist_starts, d.global_tokens, d.copy_len, 2, 8)
    with pytest.raises(taco.TacoError):
        taco.check_device()
    assert num.cpu().tolist() == [0]
