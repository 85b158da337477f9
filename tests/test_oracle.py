"""Pins of the CPU oracle against things other than itself (CPU only).

Each test fixes the oracle to a closed form, a library routine (torch's fp64 scaled-dot-product
attention), an invariant of paging, or a pure-Python brute force, so that a dropped term, a wrong sign
or index, a mis-mapped GQA head, a reversed mask bit order or a wrong block-table walk fails one of them.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from paged_kv_cache_tree_b200 import workloads as wl
from tests.brute_force import brute_force_attention


def np_inputs(w):
    return dict(
        q=wl.to_numpy_bits(w.q),
        k_cache=wl.to_numpy_bits(w.k_cache),
        v_cache=wl.to_numpy_bits(w.v_cache),
        block_tables=w.block_tables.numpy(),
        context_lens=w.context_lens.numpy(),
        num_candidates=w.num_candidates.numpy(),
        tree_mask_bits=wl.as_uint32(w.tree_mask),
        scale=w.scale,
        dtype=w.dtype,
    )


def small_spec(**kw):
    spec = dict(dtype="bf16", B=3, Hq=4, Hkv=2, D=16, bs=4, C=4, tree="forest", ctx=("uniform", 5, 23))
    spec.update(kw)
    return spec


def test_tiny_workload_shape_and_recipe():
    w = wl.make_workload("tiny")
    assert w.dtype == "fp16" and w.num_blocks == 40
    assert w.context_lens.tolist() == [37, 100]
    # chain masks: row i sees candidates 0..i
    assert [m & 0xFFFFFFFF for m in w.tree_mask[0].tolist()] == [1, 3, 7, 15]
    used = [b for b in w.block_tables.flatten().tolist() if b >= 0]
    assert len(used) == 3 + 7 and len(set(used)) == len(used)
    assert all(0 <= b < 40 for b in used)


def test_forest_masks_are_ancestor_sets():
    # parents [-1, 0, 0, 1, -1]: 0 root, 1 and 2 children of 0, 3 child of 1, 4 a second root
    masks = wl.masks_from_parents([-1, 0, 0, 1, -1], 5)
    assert masks == [0b00001, 0b00011, 0b00101, 0b01011, 0b10000]
    assert wl.masks_from_parents([-1, 0, 0, 1, -1], 3)[3:] == [0, 0]


def test_brute_force_agrees_on_tiny_shapes():
    for seed in range(3):
        for dtype in ("bf16", "fp16"):
            w = wl.make_workload(small_spec(dtype=dtype, D=8), seed=seed,
                                 num_candidates=[4, 2, 3] if seed == 1 else None)
            a = np_inputs(w)
            got = oracle.paged_tree_attention(**a)
            ref = np.array(brute_force_attention(a["q"], a["k_cache"], a["v_cache"], a["block_tables"],
                                                 a["context_lens"], a["num_candidates"],
                                                 a["tree_mask_bits"], a["scale"], dtype))
            np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def _contiguous_kv(w, b, L):
    """K, V of sequence b as [Hkv, L, D] float64, gathered with torch advanced indexing."""
    pos = torch.arange(L)
    blocks = w.block_tables[b].long()[pos // w.bs]
    slots = pos % w.bs
    K = w.k_cache.double()[blocks, :, slots, :].permute(1, 0, 2)
    V = w.v_cache.double()[blocks, :, slots, :].permute(1, 0, 2)
    return K, V


def test_chain_mask_equals_bottom_right_causal_sdpa():
    for dtype in ("bf16", "fp16"):
        w = wl.make_workload(small_spec(dtype=dtype, tree="chain", B=2, Hq=6, Hkv=2, D=16, C=5,
                                        ctx=("uniform", 9, 40)), seed=7)
        got = oracle.paged_tree_attention(**np_inputs(w))
        for b in range(w.B):
            L, n = int(w.context_lens[b]), int(w.num_candidates[b])
            P = L - n
            K, V = _contiguous_kv(w, b, L)
            Q = w.q[b, :n].double().permute(1, 0, 2)                    # [Hq, n, D]
            causal = torch.ones(n, L, dtype=torch.bool).tril(diagonal=P)  # row i sees p <= P + i
            ref = F.scaled_dot_product_attention(Q, K, V, attn_mask=causal, scale=w.scale,
                                                 enable_gqa=True)         # [Hq, n, D]
            np.testing.assert_allclose(got[b, :n], ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)


def test_single_candidate_equals_plain_decode_sdpa():
    w = wl.make_workload(small_spec(C=1, Hq=8, Hkv=2, ctx=("uniform", 1, 30)), seed=3)
    got = oracle.paged_tree_attention(**np_inputs(w))
    for b in range(w.B):
        L = int(w.context_lens[b])
        K, V = _contiguous_kv(w, b, L)
        Q = w.q[b, :1].double().permute(1, 0, 2)
        ref = F.scaled_dot_product_attention(Q, K, V, scale=w.scale, enable_gqa=True)
        np.testing.assert_allclose(got[b, :1], ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)


def test_block_permutation_invariance_is_bitwise():
    w = wl.make_workload(small_spec(), seed=11)
    a = np_inputs(w)
    base = oracle.paged_tree_attention(**a)
    rng = np.random.default_rng(5)
    perm = rng.permutation(w.num_blocks)            # old block id -> new block id
    kc = np.empty_like(a["k_cache"])
    vc = np.empty_like(a["v_cache"])
    kc[perm] = a["k_cache"]
    vc[perm] = a["v_cache"]
    bt = np.where(a["block_tables"] >= 0, perm[np.maximum(a["block_tables"], 0)], -1)
    moved = oracle.paged_tree_attention(**{**a, "k_cache": kc, "v_cache": vc, "block_tables": bt})
    assert np.array_equal(base.view(np.uint64), moved.view(np.uint64))


def test_one_key_context_returns_v_exactly():
    w = wl.make_workload(small_spec(B=2, C=1, ctx=("fixed", [1, 1])), seed=2)
    a = np_inputs(w)
    got = oracle.paged_tree_attention(**a)
    for b in range(2):
        blk = int(w.block_tables[b, 0])
        for h in range(w.Hq):
            v0 = oracle.widen_to_f64(a["v_cache"][blk, h // w.G, 0], w.dtype)
            assert np.array_equal(got[b, 0, h], v0)


def _visible_list(L, n, i, mask):
    P = L - n
    return list(range(P)) + [P + j for j in range(n) if (mask >> j) & 1]


def test_equal_keys_give_mean_of_visible_values():
    w = wl.make_workload(small_spec(), seed=4)
    a = np_inputs(w)
    kc = a["k_cache"].copy()
    kc[:] = kc[0, 0, 0]                              # every key row identical
    got = oracle.paged_tree_attention(**{**a, "k_cache": kc})
    for b in range(w.B):
        L, n = int(w.context_lens[b]), int(w.num_candidates[b])
        K, V = _contiguous_kv(w, b, L)
        for i in range(n):
            vis = _visible_list(L, n, i, int(a["tree_mask_bits"][b, i]))
            for h in range(w.Hq):
                expect = V[h // w.G, vis].mean(0).numpy()
                np.testing.assert_allclose(got[b, i, h], expect, rtol=1e-12, atol=1e-12)


def test_scale_zero_gives_mean_of_visible_values():
    w = wl.make_workload(small_spec(), seed=6)
    a = np_inputs(w)
    got = oracle.paged_tree_attention(**{**a, "scale": 0.0})
    for b in range(w.B):
        L, n = int(w.context_lens[b]), int(w.num_candidates[b])
        K, V = _contiguous_kv(w, b, L)
        for i in range(n):
            vis = _visible_list(L, n, i, int(a["tree_mask_bits"][b, i]))
            for h in range(w.Hq):
                np.testing.assert_allclose(got[b, i, h], V[h // w.G, vis].mean(0).numpy(),
                                           rtol=1e-12, atol=1e-12)


def test_two_key_closed_form():
    # one sequence, one head, D = 2, prefix of one key plus one candidate seeing itself:
    # weights e^{s0}, e^{s1} with s = scale * q.k, out = (e^{s0} v0 + e^{s1} v1) / (e^{s0} + e^{s1})
    spec = dict(dtype="bf16", B=1, Hq=1, Hkv=1, D=2, bs=2, C=1, tree="chain", ctx=("fixed", [2]))
    w = wl.make_workload(spec, seed=0)
    blk = int(w.block_tables[0, 0])
    w.q[0, 0, 0] = torch.tensor([1.0, 0.5])
    w.k_cache[blk, 0, 0] = torch.tensor([2.0, 0.0])
    w.k_cache[blk, 0, 1] = torch.tensor([-1.0, 4.0])
    w.v_cache[blk, 0, 0] = torch.tensor([3.0, -1.0])
    w.v_cache[blk, 0, 1] = torch.tensor([0.25, 8.0])
    a = np_inputs(w)
    a["scale"] = 0.5
    got = oracle.paged_tree_attention(**a)[0, 0, 0]
    s0, s1 = 0.5 * (2.0 + 0.0), 0.5 * (-1.0 + 2.0)
    e0, e1 = math.exp(s0), math.exp(s1)
    expect = [(e0 * 3.0 + e1 * 0.25) / (e0 + e1), (e0 * -1.0 + e1 * 8.0) / (e0 + e1)]
    np.testing.assert_allclose(got, expect, rtol=1e-14)


def test_only_ancestors_matter():
    w = wl.make_workload(small_spec(B=1, C=5, ctx=("fixed", [14])), seed=9,
                         parents=[[-1, 0, 0, 1, -1]])
    a = np_inputs(w)
    base = oracle.paged_tree_attention(**a)
    L, n = 14, 5
    P = L - n
    # candidate 2 is an ancestor of no row but itself: perturb its K and V
    kc, vc = a["k_cache"].copy(), a["v_cache"].copy()
    blk, slot = int(w.block_tables[0, (P + 2) // w.bs]), (P + 2) % w.bs
    kc[blk, :, slot] ^= 0x0100
    vc[blk, :, slot] ^= 0x0100
    moved = oracle.paged_tree_attention(**{**a, "k_cache": kc, "v_cache": vc})
    for i in range(n):
        same = np.array_equal(base[0, i].view(np.uint64), moved[0, i].view(np.uint64))
        assert same == (i != 2), i


def test_padding_rows_and_empty_rows_are_zero():
    w = wl.make_workload(small_spec(B=2, C=4, ctx=("fixed", [3, 9])), seed=1, num_candidates=[3, 2])
    a = np_inputs(w)
    masks = a["tree_mask_bits"].copy()
    masks[0, 1] = 0                                  # P = 0 and no candidate visible -> empty set
    got = oracle.paged_tree_attention(**{**a, "tree_mask_bits": masks})
    assert np.all(got[0, 1] == 0.0)
    assert np.all(got[0, 3] == 0.0) and np.all(got[1, 2:] == 0.0)
    assert np.all(np.isfinite(got))


def test_mask_bits_beyond_candidate_count_are_ignored():
    w = wl.make_workload(small_spec(), seed=12, num_candidates=[2, 4, 3])
    a = np_inputs(w)
    base = oracle.paged_tree_attention(**a)
    masks = a["tree_mask_bits"].copy()
    for b in range(w.B):
        n = int(w.num_candidates[b])
        masks[b, :n] |= np.uint32(0xFFFFFFFF) << np.uint32(n) if n < 32 else np.uint32(0)
    other = oracle.paged_tree_attention(**{**a, "tree_mask_bits": masks})
    assert np.array_equal(base.view(np.uint64), other.view(np.uint64))


def test_sampled_rows_match_full_evaluation():
    w = wl.make_workload(small_spec(), seed=13)
    a = np_inputs(w)
    full = oracle.paged_tree_attention(**a)
    rows = [(0, 0, 1), (2, 3, 0), (1, 1, 3)]
    part = oracle.paged_tree_attention(**a, rows=rows)
    for (b, i, h) in rows:
        assert np.array_equal(part[b, i, h], full[b, i, h])


def test_append_round_trip_and_untouched_bytes():
    w = wl.make_workload(small_spec(B=3, C=4, bs=4), seed=21, candidates_in_cache=False,
                         num_candidates=[4, 1, 0])
    kc0, vc0 = wl.to_numpy_bits(w.k_cache), wl.to_numpy_bits(w.v_cache)
    kn, vn = wl.to_numpy_bits(w.k_new), wl.to_numpy_bits(w.v_new)
    bt, so = w.block_tables.numpy(), w.slot_offsets.numpy()
    kc, vc = oracle.paged_kv_append(kn, vn, bt, so, kc0, vc0)
    # independent addressing: flatten the cache to rows [(block * Hkv + h) * bs + slot]
    written = np.zeros(kc.shape[:3], dtype=bool)
    for b in range(w.B):
        for i in range(w.C):
            s = int(so[b, i])
            if s < 0:
                continue
            blk = bt[b][s // w.bs]
            for h in range(w.Hkv):
                flat = (blk * w.Hkv + h) * w.bs + s % w.bs
                assert np.array_equal(kc.reshape(-1, w.D)[flat], kn[b, i, h])
                assert np.array_equal(vc.reshape(-1, w.D)[flat], vn[b, i, h])
                written.reshape(-1)[flat] = True
    assert int(written.sum()) == int(w.num_candidates.sum()) * w.Hkv
    # every other 16-bit word is unchanged (NaN patterns included, compared as bits)
    assert np.array_equal(kc[~written], kc0[~written]) and np.array_equal(vc[~written], vc0[~written])


def test_append_then_attend_matches_cache_prepared_with_candidates():
    spec = small_spec()
    w_cold = wl.make_workload(spec, seed=31, candidates_in_cache=False)
    w_warm = wl.make_workload(spec, seed=31, candidates_in_cache=True)
    a = np_inputs(w_cold)
    kc, vc = oracle.paged_kv_append(wl.to_numpy_bits(w_cold.k_new), wl.to_numpy_bits(w_cold.v_new),
                                    a["block_tables"], w_cold.slot_offsets.numpy(), a["k_cache"], a["v_cache"])
    got = oracle.paged_tree_attention(**{**a, "k_cache": kc, "v_cache": vc})
    ref = oracle.paged_tree_attention(**np_inputs(w_warm))
    assert np.array_equal(got.view(np.uint64), ref.view(np.uint64))


def test_tolerance_rule():
    ref = np.array([0.0, 1.0, -2.0, 100.0])
    ok = oracle.within_tolerance(ref + np.array([0.0099, 0.0299, -0.0499, 2.0099]), ref)
    bad = oracle.within_tolerance(ref + np.array([0.0101, 0.0301, 0.0501, 2.02]), ref)
    assert ok.all() and not bad.any()
    assert not oracle.within_tolerance(np.array([np.nan]), np.array([0.0])).any()
