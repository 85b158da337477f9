"""GPU parity of the acceptance step (tree masks, argmax, greedy acceptance, compaction) against the
CPU oracle: every output is an integer, so every comparison is bit-exact (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import tree_accept as ta
import paged_kv_cache_tree_b200 as taco
from paged_kv_cache_tree_b200 import workloads as wl
from tests.parity_util import gpu_step, oracle_step

pytestmark = pytest.mark.gpu


def random_forests(rng, B, C):
    par = np.full((B, C), -1, dtype=np.int32)
    for b in range(B):
        for i in range(1, C):
            par[b, i] = int(rng.integers(-1, i))
    return par


@pytest.mark.parametrize("C", [1, 5, 16, 32])
def test_masks_from_parents_bit_exact(C):
    rng = np.random.default_rng(C)
    B = 64
    par = random_forests(rng, B, C)
    par[0] = np.arange(C) - 1                      # a chain
    n = rng.integers(0, C + 1, B).astype(np.int32)
    n[:2] = C
    got = taco.tree_mask_from_parents(torch.from_numpy(par).cuda(), torch.from_numpy(n).cuda())
    assert taco.check_device() == 0
    want = ta.tree_masks(par, n)
    assert np.array_equal(got.cpu().numpy().view(np.uint32), want)


def oracle_argmax(logits: torch.Tensor, dtype: str) -> np.ndarray:
    V = logits.shape[-1]
    x = oracle.widen_to_f64(wl.to_numpy_bits(logits.cpu()), dtype).reshape(-1, V)
    return ta.logits_argmax(x)


def test_argmax_full_vocabulary_bit_exact_and_finds_the_planted_index():
    spec = dict(dtype="bf16", B=4, Hq=64, Hkv=8, D=128, bs=32, C=16, tree="forest", ctx=("fixed", [40, 60, 80, 100]))
    w = wl.make_workload(spec, seed=11, fill="zero")
    a = wl.make_accept_inputs(w)
    got = taco.logits_argmax(a.target_logits.cuda()).cpu().numpy().reshape(-1)
    assert np.array_equal(got, oracle_argmax(a.target_logits, "bf16"))
    assert np.array_equal(got, a.planted.numpy().reshape(-1))


@pytest.mark.parametrize("dtype,V,offset", [("bf16", 128256, 0), ("fp16", 32000, 0), ("bf16", 1001, 0),
                                            ("fp16", 4096, 1), ("bf16", 128256, 1), ("bf16", 8, 0), ("bf16", 1, 0)])
def test_argmax_ties_nans_and_infinities(dtype, V, offset):
    g = torch.Generator().manual_seed(V + offset)
    rows = 24
    full = torch.randint(-3, 4, (rows * V + offset,), generator=g).to(wl.TORCH_DTYPES[dtype])
    x = full[offset:].view(rows, V)
    x[1] = float("nan")
    x[2] = float("-inf")
    if V > 3:
        x[3, :3] = float("nan")
        x[4, V - 1] = float("inf")
        x[5, 0] = float("inf")
        x[5, V - 1] = float("inf")
    full[offset:] = x.reshape(-1)
    xd = full.cuda()[offset:].view(rows, V)    # offset 1: not 16-byte aligned (the scalar kernel)
    assert (xd.data_ptr() % 16 != 0) == (offset != 0)
    got = taco.logits_argmax(xd).cpu().numpy()
    assert np.array_equal(got, oracle_argmax(x.contiguous(), dtype))


@pytest.mark.parametrize("hit", [0.0, 0.5, 0.9, 1.0])
@pytest.mark.parametrize("name", ["chain", "tree"])
def test_accept_bit_exact_on_generated_trees(name, hit):
    base = dict(wl.WORKLOADS[name])
    spec = dict(base, B=12, ctx=("uniform", 20, 300))
    w = wl.make_workload(spec, seed=int(hit * 10) + 31, fill="zero", num_candidates=None)
    a = wl.make_accept_inputs(w, vocab=4096, hit_prob=hit, ties=True)
    d = w.to("cuda")
    amax = taco.logits_argmax(a.target_logits.cuda())
    got = taco.tree_greedy_accept(amax, a.tokens.cuda(), d.parents, d.num_candidates, d.context_lens)
    assert taco.check_device() == 0
    want_amax = oracle_argmax(a.target_logits, w.dtype).reshape(w.B, w.C + 1)
    assert np.array_equal(amax.cpu().numpy(), want_amax)
    want = ta.greedy_accept(want_amax, a.tokens.numpy(), w.parents.numpy(), w.num_candidates.numpy(),
                            w.context_lens.numpy())
    for g_, w_ in zip(got, want):
        assert np.array_equal(g_.cpu().numpy(), w_)


def test_accept_random_forests_small_vocabulary():
    rng = np.random.default_rng(5)
    for C in (1, 7, 32):
        B = 48
        par = random_forests(rng, B, C)
        n = rng.integers(0, C + 1, B).astype(np.int32)
        L = (n + rng.integers(0, 50, B)).astype(np.int32)
        amax = rng.integers(0, 3, (B, C + 1)).astype(np.int32)
        tok = rng.integers(0, 3, (B, C)).astype(np.int32)
        t = lambda x: torch.from_numpy(x).cuda()
        got = taco.tree_greedy_accept(t(amax), t(tok), t(par), t(n), t(L))
        assert taco.check_device() == 0
        want = ta.greedy_accept(amax, tok, par, n, L)
        for g_, w_ in zip(got, want):
            assert np.array_equal(g_.cpu().numpy(), w_)


def test_verify_then_accept_then_compact_end_to_end():
    spec = dict(dtype="bf16", B=6, Hq=32, Hkv=8, D=128, bs=16, C=8, tree="forest", ctx=("uniform", 30, 200))
    w = wl.make_workload(spec, seed=77, candidates_in_cache=False)
    out, kc, vc = gpu_step(w)                      # append the candidates, then verify
    a = wl.make_accept_inputs(w, vocab=2048, hit_prob=0.8)
    d = w.to("cuda")
    amax = taco.logits_argmax(a.target_logits.cuda())
    acc, path, bonus, slots = taco.tree_greedy_accept(amax, a.tokens.cuda(), d.parents, d.num_candidates,
                                                      d.context_lens)
    taco.paged_kv_append(d.k_new, d.v_new, d.block_tables, slots, kc, vc)
    assert taco.check_device() == 0
    _, rkc, rvc = oracle_step(w)
    want = ta.greedy_accept(a.planted.numpy(), a.tokens.numpy(), w.parents.numpy(), w.num_candidates.numpy(),
                            w.context_lens.numpy())
    rkc, rvc = oracle.paged_kv_append(wl.to_numpy_bits(w.k_new), wl.to_numpy_bits(w.v_new), w.block_tables.numpy(),
                                      want[3], rkc, rvc)
    assert np.array_equal(wl.to_numpy_bits(kc.cpu()), rkc)
    assert np.array_equal(wl.to_numpy_bits(vc.cpu()), rvc)
    assert int(want[0].sum()) > 0


def test_bad_parent_is_reported_not_faulted():
    par = torch.tensor([[-1, 0, 5, 1]], dtype=torch.int32, device="cuda")   # 5 >= 2: not an earlier candidate
    n = torch.tensor([4], dtype=torch.int32, device="cuda")
    taco.tree_mask_from_parents(par, n)
    with pytest.raises(taco.TacoError) as ei:
        taco.check_device()
    assert "parent" in str(ei.value)
    amax = torch.zeros(1, 5, dtype=torch.int32, device="cuda")
    tok = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    taco.tree_greedy_accept(amax, tok, par, n, torch.tensor([10], dtype=torch.int32, device="cuda"))
    with pytest.raises(taco.TacoError):
        taco.check_device()
    assert taco.check_device() == 0


def test_argmax_signed_zeros_tie_and_maxima_anywhere_in_the_row():
    """-0 and +0 are equal (the first wins); maxima planted across a full-vocabulary row, two per row
    (the smaller index must win)."""
    V = 128256
    rows = 40
    x = torch.full((rows, V), -1.0, dtype=torch.bfloat16)
    x[0, :] = -0.0
    x[0, 7] = 0.0
    x[1, 5] = 0.0
    x[1, 3] = -0.0
    for r in range(2, rows):
        x[r, (r * V) // (rows - 2) % V] = 2.0
        x[r, ((r * 7919) % V)] = 2.0              # a second maximum: the smaller index must win
    got = taco.logits_argmax(x.cuda()).cpu().numpy()
    assert np.array_equal(got, oracle_argmax(x, "bf16"))
    assert got[0] == 0 and got[1] == 3
    # the scratch is left clean: the same call again gives the same answer
    assert np.array_equal(taco.logits_argmax(x.cuda()).cpu().numpy(), got)


@pytest.mark.parametrize("rows", [1, 3, 16, 64, 128, 300, 2000])
def test_argmax_many_row_counts_ties_far_apart(rows):
    """Random rows of the full vocabulary, from one row to more rows than SMs: equal maxima at two
    neighbouring positions (spread over the row) or far apart, where the smaller index must win, and
    single maxima in the last or the first element."""
    V = 128256
    nvec = V // 8
    edges = sorted({k * ((nvec + s - 1) // s) * 8 for s in (2, 4, 8) for k in range(1, s)})
    g = torch.Generator().manual_seed(rows)
    x = (torch.rand(rows, V, generator=g) * 2 - 1).to(torch.bfloat16)
    for r in range(rows):
        kind = r % 4
        if kind == 0:
            e = edges[(r // 4) % len(edges)]
            x[r, e - 1] = 3.0
            x[r, e] = 3.0              # the chunk before the edge must win
        elif kind == 1:
            x[r, V - 1] = 3.0
        elif kind == 2:
            x[r, 0] = 3.0
        else:
            e = edges[(r // 4) % len(edges)]
            x[r, e] = 3.0
            x[r, V - 1] = 3.0          # the same value later in the row loses
    got = taco.logits_argmax(x.cuda()).cpu().numpy()
    want = oracle_argmax(x, "bf16")
    assert np.array_equal(got, want)
