"""GPU parity of the C-ABI path against the CPU oracle on seeded inputs (needs a B200).

Integer / byte work (the append, block-table addressing) must be bit-exact; attention rows must lie
within |gpu - ref| <= 1e-2 + 2e-2 |ref| of the fp64 oracle, padding rows must be exact zeros.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_tree_b200 as taco
from paged_kv_cache_tree_b200 import workloads as wl
from tests.parity_util import as_f64, assert_parity, full_size_rows, gpu_step, oracle_inputs, oracle_step

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _reset_options():
    taco.set_option(taco.TACO_OPT_GRID_CTAS, 0)
    taco.set_option(taco.TACO_OPT_KERNEL, 0)
    taco.set_option(taco.TACO_OPT_SEG_COST, -1)
    taco.set_option(taco.TACO_OPT_COMBINE, 0)
    yield
    taco.set_option(taco.TACO_OPT_GRID_CTAS, 0)
    taco.set_option(taco.TACO_OPT_KERNEL, 0)
    taco.set_option(taco.TACO_OPT_SEG_COST, -1)
    taco.set_option(taco.TACO_OPT_COMBINE, 0)


def test_tiny_step_append_then_attend():
    w = wl.make_workload("tiny", candidates_in_cache=False)
    out, kc, vc = gpu_step(w)
    ref, rkc, rvc = oracle_step(w)
    assert np.array_equal(wl.to_numpy_bits(kc.cpu()), rkc)
    assert np.array_equal(wl.to_numpy_bits(vc.cpu()), rvc)
    assert_parity(out, ref, w)


SMALL_CASES = [
    # dtype, B, Hq, Hkv, D, bs, C, tree, ctx, num_candidates
    ("bf16", 3, 8, 2, 128, 16, 4, "forest", ("uniform", 5, 300), None),
    ("fp16", 3, 8, 2, 128, 16, 4, "chain", ("uniform", 5, 300), None),
    ("bf16", 2, 4, 4, 64, 8, 3, "forest", ("uniform", 3, 200), None),
    ("bf16", 4, 16, 2, 128, 32, 8, "forest", ("uniform", 8, 333), [8, 1, 5, 0]),
    ("fp16", 2, 64, 8, 128, 64, 1, "chain", ("fixed", [1, 257]), None),
    ("bf16", 2, 64, 8, 128, 128, 16, "forest", ("fixed", [16, 190]), None),
    ("bf16", 3, 32, 8, 128, 16, 4, "forest", ("fixed", [64, 65, 128]), None),
    ("bf16", 2, 8, 1, 128, 256, 32, "forest", ("fixed", [40, 300]), [32, 17]),
    ("fp16", 2, 6, 2, 64, 16, 5, "chain", ("fixed", [0, 77]), [0, 5]),
    ("bf16", 5, 4, 1, 128, 16, 2, "chain", ("fixed", [2, 15, 16, 17, 63]), None),
]


KERNELS = [1, 2]   # 1 = mma.sync path, 2 = tcgen05 path (forced, whatever the tile width)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("case", range(len(SMALL_CASES)))
def test_small_shapes_full_oracle(case, kernel):
    dtype, B, Hq, Hkv, D, bs, C, tree, ctx, ncand = SMALL_CASES[case]
    spec = dict(dtype=dtype, B=B, Hq=Hq, Hkv=Hkv, D=D, bs=bs, C=C, tree=tree, ctx=ctx)
    taco.set_option(taco.TACO_OPT_KERNEL, kernel)
    w = wl.make_workload(spec, seed=100 + case, candidates_in_cache=False, num_candidates=ncand)
    out, kc, vc = gpu_step(w)
    ref, rkc, rvc = oracle_step(w)
    assert np.array_equal(wl.to_numpy_bits(kc.cpu()), rkc)
    assert np.array_equal(wl.to_numpy_bits(vc.cpu()), rvc)
    assert_parity(out, ref, w)


@pytest.mark.parametrize("kernel,combine", [(1, 1), (1, 2), (2, 1), (2, 2)])
@pytest.mark.parametrize("grid", [1, 3, 7, 64, 500])
def test_split_kv_partitions_agree(grid, kernel, combine):
    """Forced grids split the units into 1 to hundreds of pieces; either kernel's pieces are merged inside
    the verify (combine 1) or by the separate combine kernel (combine 2)."""
    spec = dict(dtype="bf16", B=3, Hq=32, Hkv=4, D=128, bs=16, C=6, tree="forest", ctx=("uniform", 100, 900))
    w = wl.make_workload(spec, seed=7)
    ref, _, _ = oracle_step(w, append=False)
    taco.set_option(taco.TACO_OPT_GRID_CTAS, grid)
    taco.set_option(taco.TACO_OPT_KERNEL, kernel)
    taco.set_option(taco.TACO_OPT_COMBINE, combine)
    out, _, _ = gpu_step(w, append=False)
    assert_parity(out, ref, w)
    again, _, _ = gpu_step(w, append=False)
    assert torch.equal(out.view(torch.int16), again.view(torch.int16)), "not deterministic run to run"


@pytest.mark.parametrize("kernel,combine", [(1, 1), (1, 2), (2, 1), (2, 2)])
@pytest.mark.parametrize("grid", [1, 5, 37, 300])
@pytest.mark.parametrize("seg_cost", [0, 1, 3, 64])
def test_weighted_work_split_agrees(seg_cost, grid, kernel, combine):
    """The work split counts seg_cost extra tiles per unit. Units of one tile next to long ones, and a
    cost far above the tiles of most units (whole CTA ranges then fall on no real tile), must still give
    every piece to exactly one CTA and merge it once."""
    spec = dict(dtype="bf16", B=10, Hq=16, Hkv=2, D=128, bs=16, C=4, tree="chain",
                ctx=("fixed", [4, 5, 17, 64, 65, 700, 6, 1500, 130, 9]))
    w = wl.make_workload(spec, seed=17)
    ref, _, _ = oracle_step(w, append=False)
    taco.set_option(taco.TACO_OPT_GRID_CTAS, grid)
    taco.set_option(taco.TACO_OPT_KERNEL, kernel)
    taco.set_option(taco.TACO_OPT_SEG_COST, seg_cost)
    taco.set_option(taco.TACO_OPT_COMBINE, combine)
    out, _, _ = gpu_step(w, append=False)
    assert_parity(out, ref, w)
    again, _, _ = gpu_step(w, append=False)
    assert torch.equal(out.view(torch.int16), again.view(torch.int16)), "not deterministic run to run"


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("grid", [0, 5])
def test_query_magnitudes_far_from_one(kernel, grid):
    """Query rows scaled by 2^40 and 2^-40, one huge element, one zero row: logits of 2^40 leave a
    float32 ulp of 2^16, so any step that adds log2 of a softmax sum to a maximum would lose the sum.
    The split grid runs the partials and their merge on the same rows."""
    spec = dict(dtype="bf16", B=2, Hq=64, Hkv=8, D=128, bs=16, C=8, tree="forest", ctx=("fixed", [300, 700]))
    w = wl.make_workload(spec, seed=8)
    q = w.q.float()
    q[0, 0, 0] *= 2.0 ** 40
    q[0, 0, 1] *= 2.0 ** -40
    q[0, 1, 2] *= 2.0 ** 20
    q[1, 0, 3] = 0.0
    q[1, 0, 4, 7] = 3e4
    q[1, 2, 9] *= 2.0 ** 30
    w.q = q.to(torch.bfloat16)
    ref, _, _ = oracle_step(w, append=False)
    taco.set_option(taco.TACO_OPT_GRID_CTAS, grid)
    taco.set_option(taco.TACO_OPT_KERNEL, kernel)
    out, _, _ = gpu_step(w, append=False)
    assert_parity(out, ref, w)


@pytest.mark.parametrize("kernel", KERNELS)
def test_block_permutation_gives_bitwise_identical_output(kernel):
    taco.set_option(taco.TACO_OPT_KERNEL, kernel)
    spec = dict(dtype="bf16", B=4, Hq=32, Hkv=8, D=128, bs=16, C=4, tree="forest", ctx=("uniform", 50, 600))
    w = wl.make_workload(spec, seed=17)
    out1, _, _ = gpu_step(w, append=False)
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(3))
    w2 = wl.make_workload(spec, seed=17)
    w2.k_cache = torch.empty_like(w.k_cache)
    w2.v_cache = torch.empty_like(w.v_cache)
    w2.k_cache[perm] = w.k_cache
    w2.v_cache[perm] = w.v_cache
    bt = w.block_tables.clone()
    mapped = bt >= 0
    bt[mapped] = perm[bt[mapped].long()].to(torch.int32)
    w2.block_tables = bt
    out2, _, _ = gpu_step(w2, append=False)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


@pytest.mark.parametrize("kernel", KERNELS)
def test_only_ancestors_matter_on_gpu(kernel):
    taco.set_option(taco.TACO_OPT_KERNEL, kernel)
    spec = dict(dtype="bf16", B=1, Hq=8, Hkv=2, D=128, bs=16, C=5, tree="chain", ctx=("fixed", [90]))
    w = wl.make_workload(spec, seed=23, parents=[[-1, 0, 0, 1, -1]])
    out1, _, _ = gpu_step(w, append=False)
    P = 90 - 5
    blk, slot = int(w.block_tables[0, (P + 2) // 16]), (P + 2) % 16
    w.k_cache[blk, :, slot] = w.k_cache[blk, :, slot] * 3 + 1
    w.v_cache[blk, :, slot] = w.v_cache[blk, :, slot] * -2
    out2, _, _ = gpu_step(w, append=False)
    for i in range(5):
        same = torch.equal(out1[0, i].view(torch.int16), out2[0, i].view(torch.int16))
        assert same == (i != 2), i


@pytest.mark.parametrize("kernel", KERNELS)
def test_one_key_context_returns_v_exactly(kernel):
    taco.set_option(taco.TACO_OPT_KERNEL, kernel)
    spec = dict(dtype="bf16", B=3, Hq=8, Hkv=2, D=128, bs=16, C=1, tree="chain", ctx=("fixed", [1, 1, 1]))
    w = wl.make_workload(spec, seed=5)
    out, _, _ = gpu_step(w, append=False)
    for b in range(3):
        blk = int(w.block_tables[b, 0])
        for h in range(8):
            assert torch.equal(out[b, 0, h].view(torch.int16), w.v_cache[blk, h // 4, 0].view(torch.int16))


@pytest.mark.parametrize("name", ["decode", "chain", "tree", "long"])
def test_full_size_workloads_sampled_rows(name):
    w = wl.make_workload(name, candidates_in_cache=False)
    out, kc, vc = gpu_step(w)
    # append: compare the written slots bit for bit against the new rows
    bt, so = w.block_tables, w.slot_offsets
    kc_cpu = kc.cpu()
    for b in range(w.B):
        for i in range(int(w.num_candidates[b])):
            s = int(so[b, i])
            blk = int(bt[b, s // w.bs])
            assert torch.equal(kc_cpu[blk, :, s % w.bs].view(torch.int16), w.k_new[b, i].view(torch.int16))
    del kc_cpu
    rows = full_size_rows(w, seed=0)
    w_after = wl.make_workload(name, candidates_in_cache=True)
    ref, _, _ = oracle_step(w_after, append=False, rows=rows)
    assert_parity(out, ref, w, rows=rows)
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("kernel", KERNELS)
def test_device_range_errors_are_reported_not_faulted(kernel):
    taco.set_option(taco.TACO_OPT_KERNEL, kernel)
    spec = dict(dtype="bf16", B=2, Hq=8, Hkv=2, D=128, bs=16, C=2, tree="chain", ctx=("fixed", [40, 70]))
    w = wl.make_workload(spec, seed=2)
    d = w.to("cuda")
    bt = d.block_tables.clone()
    bt[1, 2] = w.num_blocks + 5                      # a mapped entry pointing past the pool
    out = torch.empty_like(d.q)
    taco.paged_tree_attention(d.q, d.k_cache, d.v_cache, bt, d.context_lens, d.num_candidates, d.tree_mask,
                              w.scale, out=out)
    with pytest.raises(taco.TacoError) as ei:
        taco.check_device()
    assert "block id" in str(ei.value)
    ctx = d.context_lens.clone()
    ctx[0] = 10 ** 6                                  # longer than the block table can map
    taco.paged_tree_attention(d.q, d.k_cache, d.v_cache, d.block_tables, ctx, d.num_candidates, d.tree_mask,
                              w.scale, out=out)
    with pytest.raises(taco.TacoError) as ei:
        taco.check_device()
    assert "context length" in str(ei.value)
    so = d.slot_offsets.clone()
    so[0, 0] = 10 ** 6
    taco.paged_kv_append(d.k_new, d.v_new, d.block_tables, so, d.k_cache, d.v_cache)
    with pytest.raises(taco.TacoError) as ei:
        taco.check_device()
    assert "slot" in str(ei.value)
    # the context is still usable and a clean call reports nothing
    taco.paged_tree_attention(d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, d.num_candidates,
                              d.tree_mask, w.scale, out=out)
    assert taco.check_device() == 0


def test_append_skips_negative_slots_and_touches_nothing_else():
    spec = dict(dtype="fp16", B=3, Hq=4, Hkv=2, D=64, bs=8, C=4, tree="chain", ctx=("fixed", [9, 30, 4]))
    w = wl.make_workload(spec, seed=8, candidates_in_cache=False, num_candidates=[4, 0, 2])
    d = w.to("cuda")
    before_k = d.k_cache.clone()
    taco.paged_kv_append(d.k_new, d.v_new, d.block_tables, d.slot_offsets, d.k_cache, d.v_cache)
    assert taco.check_device() == 0
    _, rkc, rvc = oracle_step(w)
    assert np.array_equal(wl.to_numpy_bits(d.k_cache.cpu()), rkc)
    assert np.array_equal(wl.to_numpy_bits(d.v_cache.cpu()), rvc)
    changed = (d.k_cache.view(torch.int16) != before_k.view(torch.int16)).any(dim=-1).sum().item()
    assert changed <= (4 + 2) * 2


def test_two_streams_overlap_without_sharing_a_workspace():
    """Two verifies of different shapes, both with split units, enqueued on two streams with no order
    between them: each (device, stream) pair has its own workspace and error word, so both results
    match the oracle and each stream's error check sees only its own calls."""
    specs = [dict(dtype="bf16", B=2, Hq=32, Hkv=8, D=128, bs=16, C=1, tree="chain", ctx=("uniform", 3000, 6000)),
             dict(dtype="bf16", B=2, Hq=64, Hkv=8, D=128, bs=32, C=8, tree="forest", ctx=("uniform", 3000, 6000))]
    ws = [wl.make_workload(s, seed=300 + k) for k, s in enumerate(specs)]
    ds = [w.to("cuda") for w in ws]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [torch.full_like(d.q, float("nan")) for d in ds]
    torch.cuda.synchronize()
    for rep in range(3):
        for k in range(2):
            taco.paged_tree_attention(ds[k].q, ds[k].k_cache, ds[k].v_cache, ds[k].block_tables, ds[k].context_lens,
                                      ds[k].num_candidates, ds[k].tree_mask, ws[k].scale, out=outs[k],
                                      stream=streams[k])
    # a bad block id on stream 1 only: stream 0's word stays clean
    bt = ds[1].block_tables.clone()
    bt[0, 1] = ws[1].num_blocks + 3
    bad_out = torch.empty_like(ds[1].q)
    taco.paged_tree_attention(ds[1].q, ds[1].k_cache, ds[1].v_cache, bt, ds[1].context_lens, ds[1].num_candidates,
                              ds[1].tree_mask, ws[1].scale, out=bad_out, stream=streams[1])
    assert taco.check_device(streams[0]) == 0
    with pytest.raises(taco.TacoError) as ei:
        taco.check_device(streams[1])
    assert "block id" in str(ei.value)
    torch.cuda.synchronize()
    for k in range(2):
        want, _, _ = oracle_step(ws[k], append=False)
        assert_parity(outs[k].cpu(), want, ws[k])


def test_bounded_pipeline_wait_runs_out_and_reports():
    """The first CTA's producers leave one stage unarmed (TACO_OPT_TEST_STALL, mma.sync kernel), so a
    consumer's bounded wait on it runs out: the call still returns, the stream's error word carries
    TACO_DEVERR_WAIT_TIMEOUT (reading it also clears the split-KV counters), and the next clean call
    gives the same bits as a clean call before the stall."""
    spec = dict(dtype="bf16", B=4, Hq=32, Hkv=8, D=128, bs=16, C=1, tree="chain", ctx=("uniform", 600, 1500))
    w = wl.make_workload(spec, seed=12)
    d = w.to("cuda")
    taco.set_option(taco.TACO_OPT_KERNEL, 1)
    taco.set_option(taco.TACO_OPT_GRID_CTAS, 7)   # every unit split: the counters take part too

    def call():
        out = torch.full_like(d.q, float("nan"))
        taco.paged_tree_attention(d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, d.num_candidates,
                                  d.tree_mask, w.scale, out=out)
        return out

    before = call()
    assert taco.check_device() == 0
    ref, _, _ = oracle_step(w, append=False)
    assert_parity(before.cpu(), ref, w)
    try:
        taco.set_option(taco.TACO_OPT_TEST_STALL, 2)   # CTA 0's second tile
        call()
        with pytest.raises(taco.TacoError) as ei:
            taco.check_device()
        assert "pipeline wait timed out" in str(ei.value)
    finally:
        taco.set_option(taco.TACO_OPT_TEST_STALL, 0)
    after = call()
    assert taco.check_device() == 0
    assert torch.equal(after.view(torch.int16), before.view(torch.int16))


@pytest.mark.parametrize("dtype,D,combine", [("bf16", 128, 2), ("fp16", 64, 2), ("bf16", 128, 0)])
def test_separate_combine_on_few_long_units_and_launch_count(dtype, D, combine):
    """Two sequences of thousands of keys on a full grid: every unit is cut into dozens of pieces, which
    the separate combine kernel merges (chosen automatically for so few units). The call reports its
    launches: the append kernel, the verify and the combine."""
    spec = dict(dtype=dtype, B=2, Hq=32, Hkv=4, D=D, bs=64, C=4, tree="chain", ctx=("uniform", 6000, 12000))
    w = wl.make_workload(spec, seed=21, candidates_in_cache=False)
    taco.set_option(taco.TACO_OPT_COMBINE, combine)
    d = w.to("cuda")
    out = torch.full_like(d.q, float("nan"))
    taco.paged_tree_attention_append(d.q, d.k_new, d.v_new, d.k_cache, d.v_cache, d.block_tables, d.context_lens,
                                     d.num_candidates, d.tree_mask, w.scale, out=out)
    assert taco.last_call_launches() == 3
    assert taco.check_device() == 0
    ref, _, _ = oracle_step(w)
    assert_parity(out.cpu(), ref, w)
    # the same call twice gives the same bits
    again = torch.full_like(d.q, float("nan"))
    taco.paged_tree_attention(d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, d.num_candidates,
                              d.tree_mask, w.scale, out=again)
    assert taco.last_call_launches() == 2
    assert torch.equal(out.view(torch.int16), again.view(torch.int16))
