"""GPU parity of paged_tree_attention_append (append of the candidates fused into the verify for narrow
units, append kernel first otherwise) against the oracle's paged_kv_append followed by its attention
(needs a B200). Candidate slots start NaN-poisoned, so a candidate row the kernel failed to patch would
show up in the output."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_tree_b200 as taco
from paged_kv_cache_tree_b200 import workloads as wl
from tests.parity_util import assert_parity, full_size_rows, oracle_step

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _reset_options():
    taco.set_option(taco.TACO_OPT_GRID_CTAS, 0)
    yield
    taco.set_option(taco.TACO_OPT_GRID_CTAS, 0)


def fused_step(w):
    d = w.to("cuda")
    out = torch.full_like(d.q, float("nan"))
    taco.paged_tree_attention_append(d.q, d.k_new, d.v_new, d.k_cache, d.v_cache, d.block_tables, d.context_lens,
                                     d.num_candidates, d.tree_mask, w.scale, out=out)
    assert taco.check_device() == 0
    return out.cpu(), d.k_cache.cpu(), d.v_cache.cpu()


CASES = [
    # dtype, B, Hq, Hkv, D, bs, C, tree, ctx, num_candidates      (packed rows G*C -> kernel form)
    ("bf16", 5, 32, 8, 128, 16, 1, "chain", ("uniform", 1, 700), None),        # 4: swapped, fused
    ("fp16", 4, 16, 2, 128, 16, 1, "chain", ("fixed", [1, 64, 65, 300]), None),  # 8: swapped, fused
    ("bf16", 4, 8, 4, 64, 8, 4, "forest", ("uniform", 4, 300), [4, 0, 2, 3]),   # 8: swapped D64, fused
    ("bf16", 3, 16, 4, 128, 32, 3, "forest", ("uniform", 3, 400), None),       # 12: MT=1, fused
    ("fp16", 3, 8, 2, 128, 64, 4, "chain", ("fixed", [63, 66, 200]), None),    # 16: MT=1, fused, straddles
    ("bf16", 2, 64, 8, 128, 16, 4, "chain", ("uniform", 100, 500), None),      # 32: MT=2, append kernel
    ("bf16", 2, 64, 8, 128, 32, 8, "forest", ("uniform", 50, 400), None),      # 64: tcgen05, append kernel
]


@pytest.mark.parametrize("grid", [0, 1, 7])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_fused_append_then_attention_matches_oracle(case, grid):
    dtype, B, Hq, Hkv, D, bs, C, tree, ctx, ncand = CASES[case]
    spec = dict(dtype=dtype, B=B, Hq=Hq, Hkv=Hkv, D=D, bs=bs, C=C, tree=tree, ctx=ctx)
    w = wl.make_workload(spec, seed=300 + case, candidates_in_cache=False, num_candidates=ncand)
    taco.set_option(taco.TACO_OPT_GRID_CTAS, grid)
    out, kc, vc = fused_step(w)
    ref, rkc, rvc = oracle_step(w)
    assert np.array_equal(wl.to_numpy_bits(kc), rkc)
    assert np.array_equal(wl.to_numpy_bits(vc), rvc)
    assert_parity(out, ref, w)


@pytest.mark.parametrize("name", ["decode", "chain", "tree", "long"])
def test_full_size_sampled_rows(name):
    """The bench's call at full size: decode fuses the append; chain, tree and long run the append kernel,
    and the verify waits for it only before the tiles that hold the candidates' slots."""
    w = wl.make_workload(name, candidates_in_cache=False)
    out, kc, vc = fused_step(w)
    so, bt = w.slot_offsets, w.block_tables
    for b in range(w.B):
        for i in range(int(w.num_candidates[b])):
            s = int(so[b, i])
            blk = int(bt[b, s // w.bs])
            assert torch.equal(kc[blk, :, s % w.bs].view(torch.int16), w.k_new[b, i].view(torch.int16))
            assert torch.equal(vc[blk, :, s % w.bs].view(torch.int16), w.v_new[b, i].view(torch.int16))
    rows = full_size_rows(w, seed=4)
    w_after = wl.make_workload(name, candidates_in_cache=True)
    ref, _, _ = oracle_step(w_after, append=False, rows=rows)
    assert_parity(out, ref, w, rows=rows)
    assert torch.isfinite(out.float()).all()


def test_bad_block_id_is_reported_not_faulted():
    spec = dict(dtype="bf16", B=2, Hq=32, Hkv=8, D=128, bs=16, C=1, tree="chain", ctx=("fixed", [40, 70]))
    w = wl.make_workload(spec, seed=9)
    bt = w.block_tables.clone()
    bt[1, (70 - 1) // 16] = 10 ** 6          # the candidate's block of sequence 1
    d = w.to("cuda")
    out = torch.empty_like(d.q)
    taco.paged_tree_attention_append(d.q, d.k_new, d.v_new, d.k_cache, d.v_cache, bt.cuda(), d.context_lens,
                                     d.num_candidates, d.tree_mask, w.scale, out=out)
    with pytest.raises(taco.TacoError) as ei:
        taco.check_device()
    assert "block id" in str(ei.value)
    assert taco.check_device() == 0
