"""One speculative step through every entry point, each stage checked against the CPU oracle (needs a
B200): Lookahead Cache forests -> tree masks -> fused KV-append + verify attention -> argmax of target
logits -> greedy acceptance -> compaction append of the accepted K/V -> copy_len update."""
import numpy as np
import torch

import oracle
import paged_kv_cache_tree_b200 as taco
from oracle import lookahead_cache as la
from oracle import tree_accept as ta
from paged_kv_cache_tree_b200 import workloads as wl
from tests.parity_util import assert_parity, oracle_step

import pytest

pytestmark = pytest.mark.gpu


def test_one_speculative_step_end_to_end():
    B, C, V = 6, 4, 512
    # 1. candidate forests from each sequence's history and a shared cache (small vocabulary: many matches)
    li = wl.make_lookahead_inputs(B=B, hist_len=(40, 300), n_docs=3, doc_len=(50, 300), n_phrases=12,
                                  phrase_len=(2, 5), p_phrase=0.9, vocab=V, copy_len=(2, 4), max_match=3, C=C,
                                  seed=77)
    dl = li.to("cuda")
    tok, par, num = taco.lookahead_propose(dl.history, dl.hist_starts, dl.global_tokens, dl.copy_len, li.max_match, C)
    want_tok, want_par, want_num = la.propose_batch(li.histories(), li.global_tokens.tolist(), li.max_match,
                                                    li.copy_len.numpy(), C)
    assert np.array_equal(tok.cpu().numpy(), want_tok) and np.array_equal(par.cpu().numpy(), want_par)
    assert np.array_equal(num.cpu().numpy(), want_num)
    assert want_num.sum() > 0
    # 2. tree masks
    masks = taco.tree_mask_from_parents(par, num)
    assert np.array_equal(masks.cpu().numpy().view(np.uint32), ta.tree_masks(want_par, want_num))
    # 3. the verify step over these candidates: K/V append fused into the attention (16 packed rows)
    spec = dict(dtype="bf16", B=B, Hq=32, Hkv=8, D=128, bs=16, C=C, tree="forest", ctx=("uniform", 20, 400))
    w = wl.make_workload(spec, seed=78, candidates_in_cache=False, num_candidates=want_num.tolist(),
                         parents=want_par.tolist())
    assert np.array_equal(wl.as_uint32(w.tree_mask), ta.tree_masks(want_par, want_num))
    d = w.to("cuda")
    out = torch.full_like(d.q, float("nan"))
    taco.paged_tree_attention_append(d.q, d.k_new, d.v_new, d.k_cache, d.v_cache, d.block_tables, d.context_lens,
                                     num, masks, w.scale, out=out)
    assert taco.check_device() == 0
    ref, rkc, rvc = oracle_step(w)
    assert np.array_equal(wl.to_numpy_bits(d.k_cache.cpu()), rkc)
    assert np.array_equal(wl.to_numpy_bits(d.v_cache.cpu()), rvc)
    assert_parity(out.cpu(), ref, w)
    # 4. target logits after the prefix and after each candidate: plant some candidates as the argmax
    g = torch.Generator().manual_seed(79)
    logits = torch.randn(B, C + 1, V, generator=g)
    for b in range(B):
        for i in range(int(want_num[b])):
            if float(torch.rand(1, generator=g)) < 0.7:
                row = 0 if want_par[b, i] < 0 else int(want_par[b, i]) + 1
                logits[b, row, int(want_tok[b, i])] = 10.0 + i   # later siblings win ties of planting
    logits = logits.to(torch.bfloat16)
    amax = taco.logits_argmax(logits.cuda())
    want_amax = ta.logits_argmax(oracle.widen_to_f64(wl.to_numpy_bits(logits), "bf16").reshape(-1, V)).reshape(B, C + 1)
    assert np.array_equal(amax.cpu().numpy(), want_amax)
    # 5. greedy acceptance of the proposed forests
    acc_len, path, bonus, slots = taco.tree_greedy_accept(amax, tok, par, num, d.context_lens)
    assert taco.check_device() == 0
    want = ta.greedy_accept(want_amax, want_tok, want_par, want_num, w.context_lens.numpy())
    for got_x, want_x in zip((acc_len, path, bonus, slots), want):
        assert np.array_equal(got_x.cpu().numpy(), want_x)
    # 6. the accepted candidates' K/V move to the contiguous tail
    taco.paged_kv_append(d.k_new, d.v_new, d.block_tables, slots, d.k_cache, d.v_cache)
    assert taco.check_device() == 0
    rkc, rvc = oracle.paged_kv_append(wl.to_numpy_bits(w.k_new), wl.to_numpy_bits(w.v_new), w.block_tables.numpy(),
                                      want[3], rkc, rvc)
    assert np.array_equal(wl.to_numpy_bits(d.k_cache.cpu()), rkc)
    assert np.array_equal(wl.to_numpy_bits(d.v_cache.cpu()), rvc)
    # 7. copy_len for the next step
    hit = torch.full((B,), 0.5, dtype=torch.float32, device="cuda")
    cl = torch.zeros(B, dtype=torch.int32, device="cuda")
    taco.lookahead_update_copy_len(acc_len, num, hit, cl, copy_max=8)
    want_hit, want_cl = la.update_copy_len(np.full(B, 0.5, np.float32), want[0], want_num, batch=B, copy_max=8,
                                           alpha=0.5, batch_ref=16)
    assert np.array_equal(hit.cpu().numpy().view(np.uint32), want_hit.view(np.uint32))
    assert np.array_equal(cl.cpu().numpy(), want_cl)
    assert int(want[0].sum()) > 0
