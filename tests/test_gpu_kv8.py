"""GPU parity of the e4m3 (8-bit) KV cache path against the CPU oracle (needs a B200).

The quantising append is byte work: its codes must equal the oracle's bit for bit (division in
float32, nearest e4m3 with ties to the even code, saturation at 448). The attention over e4m3 caches
must lie within |gpu - ref| <= 1e-2 + 2e-2 |ref| of the fp64 oracle that decodes the same codes.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import fp8
import paged_kv_cache_tree_b200 as taco
from paged_kv_cache_tree_b200 import workloads as wl
from tests.parity_util import assert_parity, full_size_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _reset_options():
    taco.set_option(taco.TACO_OPT_GRID_CTAS, 0)
    taco.set_option(taco.TACO_OPT_KERNEL, 0)
    yield
    taco.set_option(taco.TACO_OPT_GRID_CTAS, 0)
    taco.set_option(taco.TACO_OPT_KERNEL, 0)


def oracle_attention_e4m3(w, c8, rows=None, k_cache=None, v_cache=None):
    return oracle.paged_tree_attention(
        wl.to_numpy_bits(w.q), (c8.k_cache if k_cache is None else k_cache).numpy(),
        (c8.v_cache if v_cache is None else v_cache).numpy(), w.block_tables.numpy(), w.context_lens.numpy(),
        w.num_candidates.numpy(), wl.as_uint32(w.tree_mask), w.scale, w.dtype, rows=rows, kv_dtype="e4m3",
        k_scale=c8.k_scale.numpy(), v_scale=c8.v_scale.numpy())


def gpu_attention_e4m3(w, c8):
    d, g8 = w.to("cuda"), c8.to("cuda")
    out = torch.full_like(d.q, float("nan"))
    taco.paged_tree_attention_e4m3(d.q, g8.k_cache, g8.v_cache, g8.k_scale, g8.v_scale, d.block_tables,
                                   d.context_lens, d.num_candidates, d.tree_mask, w.scale, out=out)
    assert taco.check_device() == 0
    return out.cpu()


def special_rows(w):
    """Overwrite some new K/V rows with values that probe the rounding: exact midpoints between e4m3
    neighbours (ties go to the even code), values past 448 (saturation), +-inf, tiny values
    (subnormal codes and underflow to zero), signed zeros and NaN (both signs, through V = -row)."""
    k, v = w.k_new.clone(), w.v_new.clone()
    D = w.D
    probe = torch.tensor([1.0625, 1.1875, -1.0625, 0.3125 * 1.0625, 500.0, -1e4, float("inf"), float("-inf"),
                          2.0 ** -10, -(2.0 ** -10) * 1.5, 2.0 ** -12, 0.0, -0.0, 448.0, 464.0, 480.0, float("nan")])
    reps = (D + len(probe) - 1) // len(probe)
    row = probe.repeat(reps)[:D].to(k.dtype)
    k[0, 0, 0] = row
    v[0, 0, -1] = -row
    return k, v


@pytest.mark.parametrize("dtype,D,bs", [("bf16", 128, 16), ("fp16", 128, 32), ("bf16", 64, 8), ("fp16", 64, 64)])
def test_quantising_append_bit_exact(dtype, D, bs):
    spec = dict(dtype=dtype, B=4, Hq=8, Hkv=2, D=D, bs=bs, C=5, tree="forest", ctx=("uniform", 6, 200))
    w = wl.make_workload(spec, seed=3 + D + bs, candidates_in_cache=False, num_candidates=[5, 0, 3, 5])
    c8 = wl.make_e4m3_cache(w, seed=9)
    k_new, v_new = special_rows(w)
    scales = (torch.tensor([1.0, 0.0173] if dtype == "bf16" else [0.5, 3.7]),
              torch.tensor([0.25, 1.0] if dtype == "bf16" else [1.0, 0.011]))
    so = w.slot_offsets.clone()
    so[2, 1] = -1                                  # a skipped row
    g = {k: v.cuda() for k, v in dict(k_new=k_new, v_new=v_new, bt=w.block_tables, so=so,
                                      kc=c8.k_cache, vc=c8.v_cache).items()}
    ks, vs = scales[0].float().cuda(), scales[1].float().cuda()
    taco.paged_kv_append_e4m3(g["k_new"], g["v_new"], g["bt"], g["so"], ks, vs, g["kc"], g["vc"])
    assert taco.check_device() == 0
    rk, rv = fp8.paged_kv_append_e4m3(wl.to_numpy_bits(k_new), wl.to_numpy_bits(v_new), dtype,
                                      w.block_tables.numpy(), so.numpy(), scales[0].numpy(), scales[1].numpy(),
                                      c8.k_cache.numpy(), c8.v_cache.numpy())
    assert np.array_equal(g["kc"].cpu().numpy(), rk)
    assert np.array_equal(g["vc"].cpu().numpy(), rv)
    # the probes landed where expected (row (0, 0) sits at slot P_0)
    P0 = int(w.context_lens[0]) - int(w.num_candidates[0])
    blk = int(w.block_tables[0, P0 // bs])
    codes = g["kc"][blk, 0, P0 % bs].cpu().numpy()
    if dtype == "bf16":                            # scale 1: 1.0625 is a tie between 1.0 and 1.125
        assert codes[0] == 0x38 and codes[2] == 0xB8 and codes[4] == 0x7E and codes[6] == 0x7E
        assert codes[7] == 0xFE and codes[11] == 0x00 and codes[12] == 0x80 and codes[16] == 0x7F


SHAPES = [
    # Hq, Hkv, D, C, tree, bs, ctx
    (32, 8, 128, 1, "chain", 16, ("uniform", 1, 700)),      # decode: 4 packed rows
    (64, 8, 128, 4, "chain", 64, ("uniform", 100, 900)),    # 32 packed rows
    (64, 8, 128, 8, "forest", 32, ("uniform", 8, 500)),     # 64 packed rows (tensor-core kernel)
    (64, 8, 128, 16, "forest", 32, ("uniform", 8, 700)),    # 128 packed rows: the tree shape
    (8, 1, 128, 5, "forest", 16, ("fixed", [5, 64, 65, 129])),
    (32, 8, 64, 4, "chain", 16, ("uniform", 1, 600)),       # head_dim 64
    (64, 8, 64, 16, "forest", 8, ("uniform", 8, 400)),
]


def _mma_possible(shape):
    Hq, Hkv, D, C = shape[:4]
    return D == 128 and (Hq // Hkv) * C <= 64


@pytest.mark.parametrize("kernel,grid", [(0, 0), (0, 3), (0, 50), (1, 0), (2, 0), (2, 7)])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("shape", SHAPES)
def test_attention_over_e4m3_cache(shape, dtype, kernel, grid):
    """Every shape on the automatic choice and on each kernel that takes it (1 = mma.sync with codes
    widened in registers, 2 = tcgen05 with tiles widened once in shared memory), several grids."""
    Hq, Hkv, D, C, tree, bs, ctx = shape
    if kernel == 1 and not _mma_possible(shape):
        pytest.skip("the mma.sync e4m3 kernel takes head_dim 128 and <= 64 packed rows")
    B = 4
    spec = dict(dtype=dtype, B=B, Hq=Hq, Hkv=Hkv, D=D, bs=bs, C=C, tree=tree, ctx=ctx)
    w = wl.make_workload(spec, seed=40 + C + Hq + bs + D)
    c8 = wl.make_e4m3_cache(w)
    taco.set_option(taco.TACO_OPT_KERNEL, kernel)
    taco.set_option(taco.TACO_OPT_GRID_CTAS, grid)
    got = gpu_attention_e4m3(w, c8)
    ref = oracle_attention_e4m3(w, c8)
    assert_parity(got, ref, w)


def test_empty_contexts_and_padding_rows_are_zero():
    spec = dict(dtype="bf16", B=3, Hq=16, Hkv=4, D=128, bs=16, C=4, tree="chain", ctx=("fixed", [0, 3, 40]))
    w = wl.make_workload(spec, seed=5, num_candidates=[0, 2, 4])
    c8 = wl.make_e4m3_cache(w)
    got = gpu_attention_e4m3(w, c8)
    assert torch.all(got[0] == 0) and torch.all(got[1, 2:] == 0)
    assert_parity(got, oracle_attention_e4m3(w, c8), w)


@pytest.mark.parametrize("Hq,C", [(16, 2), (64, 8)])
def test_query_magnitudes_far_from_one(Hq, C):
    """bf16 queries with rows scaled by 2^40 .. 2^-40 and single huge or tiny elements: the kernels
    rescale each query row into f16 range by a power of two (in registers on the mma.sync kernel, 16
    packed rows; in a pre-pass on the tcgen05 kernel, 64 packed rows) and must still match."""
    spec = dict(dtype="bf16", B=2, Hq=Hq, Hkv=2 if Hq == 16 else 8, D=128, bs=16, C=C, tree="chain",
                ctx=("fixed", [90, 300]))
    w = wl.make_workload(spec, seed=8)
    q = w.q.float()
    q[0, 0, 0] *= 2.0 ** 40
    q[0, 0, 1] *= 2.0 ** -40
    q[0, 1, 2] *= 2.0 ** -12
    q[1, 0, 3] = 0.0
    q[1, 0, 4, 7] = 3e4
    q[1, 1, 5, :100] *= 2.0 ** -30
    w.q = q.to(torch.bfloat16)
    c8 = wl.make_e4m3_cache(w)
    assert_parity(gpu_attention_e4m3(w, c8), oracle_attention_e4m3(w, c8), w)


def test_append_then_attend_end_to_end():
    spec = dict(dtype="bf16", B=5, Hq=32, Hkv=8, D=128, bs=16, C=4, tree="forest", ctx=("uniform", 4, 400))
    w = wl.make_workload(spec, seed=21, candidates_in_cache=False)
    c8 = wl.make_e4m3_cache(w)
    d, g8 = w.to("cuda"), c8.to("cuda")
    taco.paged_kv_append_e4m3(d.k_new, d.v_new, d.block_tables, d.slot_offsets, g8.k_scale, g8.v_scale,
                              g8.k_cache, g8.v_cache)
    out = torch.full_like(d.q, float("nan"))
    taco.paged_tree_attention_e4m3(d.q, g8.k_cache, g8.v_cache, g8.k_scale, g8.v_scale, d.block_tables,
                                   d.context_lens, d.num_candidates, d.tree_mask, w.scale, out=out)
    assert taco.check_device() == 0
    rk, rv = fp8.paged_kv_append_e4m3(wl.to_numpy_bits(w.k_new), wl.to_numpy_bits(w.v_new), w.dtype,
                                      w.block_tables.numpy(), w.slot_offsets.numpy(), c8.k_scale.numpy(),
                                      c8.v_scale.numpy(), c8.k_cache.numpy(), c8.v_cache.numpy())
    assert np.array_equal(g8.k_cache.cpu().numpy(), rk)
    assert np.array_equal(g8.v_cache.cpu().numpy(), rv)
    ref = oracle_attention_e4m3(w, c8, k_cache=torch.from_numpy(rk), v_cache=torch.from_numpy(rv))
    assert_parity(out.cpu(), ref, w)


@pytest.mark.parametrize("name", ["decode", "chain", "tree", "long"])
def test_full_size_workloads_sampled_rows(name):
    """The bench's workloads at full size with e4m3 caches, in the default launch configuration: one row
    of every (sequence, KV head) unit plus 24 sampled rows against the oracle."""
    w = wl.make_workload(name)
    c8 = wl.make_e4m3_cache(w)
    got = gpu_attention_e4m3(w, c8)
    rows = full_size_rows(w, seed=1)
    assert_parity(got, oracle_attention_e4m3(w, c8, rows=rows), w, rows=rows)
    assert torch.isfinite(got.float()).all()


@pytest.mark.parametrize("spec", [
    dict(dtype="bf16", B=3, Hq=64, Hkv=8, D=128, bs=16, C=8, tree="chain", ctx=("uniform", 9, 900)),
    dict(dtype="fp16", B=3, Hq=32, Hkv=8, D=64, bs=32, C=4, tree="forest", ctx=("uniform", 5, 500)),
    dict(dtype="bf16", B=4, Hq=32, Hkv=8, D=128, bs=16, C=1, tree="chain", ctx=("uniform", 1, 300)),
])
def test_append_and_attend_in_one_call(spec):
    """paged_tree_attention_append_e4m3: the candidates' rows quantised into slots P_b .. L_b - 1, then
    the attention, in one call; the caches equal the quantising-append oracle byte for byte and the
    output the attention oracle over them."""
    w = wl.make_workload(spec, seed=77, candidates_in_cache=False)
    c8 = wl.make_e4m3_cache(w)
    d, g8 = w.to("cuda"), c8.to("cuda")
    out = torch.full_like(d.q, float("nan"))
    taco.paged_tree_attention_e4m3(d.q, g8.k_cache, g8.v_cache, g8.k_scale, g8.v_scale, d.block_tables,
                                   d.context_lens, d.num_candidates, d.tree_mask, w.scale, out=out,
                                   k_new=d.k_new, v_new=d.v_new)
    assert taco.check_device() == 0
    rk, rv = fp8.paged_kv_append_e4m3(wl.to_numpy_bits(w.k_new), wl.to_numpy_bits(w.v_new), w.dtype,
                                      w.block_tables.numpy(), w.slot_offsets.numpy(), c8.k_scale.numpy(),
                                      c8.v_scale.numpy(), c8.k_cache.numpy(), c8.v_cache.numpy())
    assert np.array_equal(g8.k_cache.cpu().numpy(), rk)
    assert np.array_equal(g8.v_cache.cpu().numpy(), rv)
    ref = oracle_attention_e4m3(w, c8, k_cache=torch.from_numpy(rk), v_cache=torch.from_numpy(rv))
    assert_parity(out.cpu(), ref, w)


def _one_call_e4m3(w, c8):
    d, g8 = w.to("cuda"), c8.to("cuda")
    out = torch.full_like(d.q, float("nan"))
    taco.paged_tree_attention_e4m3(d.q, g8.k_cache, g8.v_cache, g8.k_scale, g8.v_scale, d.block_tables,
                                   d.context_lens, d.num_candidates, d.tree_mask, w.scale, out=out,
                                   k_new=d.k_new, v_new=d.v_new)
    assert taco.check_device() == 0
    launches = taco.last_call_launches()
    rk, rv = fp8.paged_kv_append_e4m3(wl.to_numpy_bits(w.k_new), wl.to_numpy_bits(w.v_new), w.dtype,
                                      w.block_tables.numpy(), w.slot_offsets.numpy(), c8.k_scale.numpy(),
                                      c8.v_scale.numpy(), c8.k_cache.numpy(), c8.v_cache.numpy())
    assert np.array_equal(g8.k_cache.cpu().numpy(), rk)
    assert np.array_equal(g8.v_cache.cpu().numpy(), rv)
    return out.cpu(), rk, rv, launches


def _launches_16bit(w):
    d = w.to("cuda")
    out = torch.empty_like(d.q)
    taco.paged_tree_attention_append(d.q, d.k_new, d.v_new, d.k_cache, d.v_cache, d.block_tables, d.context_lens,
                                     d.num_candidates, d.tree_mask, w.scale, out=out)
    assert taco.check_device() == 0
    return taco.last_call_launches()


@pytest.mark.parametrize("grid", [0, 5, 300])
@pytest.mark.parametrize("spec", [
    # 16 packed rows (one 16-row tile per unit)
    dict(dtype="bf16", B=5, Hq=32, Hkv=8, D=128, bs=16, C=4, tree="forest", ctx=("uniform", 4, 700)),
    # 8 and 4 packed rows (the swapped form)
    dict(dtype="fp16", B=4, Hq=64, Hkv=8, D=128, bs=64, C=1, tree="chain", ctx=("uniform", 1, 900)),
    dict(dtype="bf16", B=4, Hq=8, Hkv=4, D=128, bs=32, C=2, tree="forest", ctx=("fixed", [2, 31, 129, 600])),
])
def test_fused_quantising_append_on_narrow_units(spec, grid):
    """Units of <= 16 packed rows quantise the candidates' rows inside the verify kernel, as the 16-bit
    path copies them: the call launches no append kernel (the same launches as the 16-bit one-call
    path), the caches equal the quantising-append oracle byte for byte (rounding probes included: ties,
    saturation, infinities, subnormals, signed zeros), and the output the attention oracle over them.
    Grids of 5 and 300 CTAs cut the units (and the candidates' tiles) into pieces."""
    w = wl.make_workload(spec, seed=90 + spec["C"] + spec["bs"], candidates_in_cache=False)
    k, v = special_rows(w)
    # NaN probes stay with the append-only tests: here every row is attended
    w.k_new, w.v_new = torch.nan_to_num(k, nan=0.75), torch.nan_to_num(v, nan=-0.75)
    c8 = wl.make_e4m3_cache(w)
    taco.set_option(taco.TACO_OPT_GRID_CTAS, grid)
    got, rk, rv, launches = _one_call_e4m3(w, c8)
    ref = oracle_attention_e4m3(w, c8, k_cache=torch.from_numpy(rk), v_cache=torch.from_numpy(rv))
    assert_parity(got, ref, w)
    assert launches == _launches_16bit(w)


@pytest.mark.parametrize("name", ["decode", "long"])
def test_full_size_one_call_sampled_rows(name):
    """paged_tree_attention_append_e4m3 on the full decode workload (the append fused into the
    verify) and on the full long workload (the append kernel, then the verify reading all but the
    appended slots before the append ends): caches byte-exact, one row of every unit plus 24 sampled
    rows against the oracle."""
    w = wl.make_workload(name, candidates_in_cache=False)
    c8 = wl.make_e4m3_cache(w)
    got, rk, rv, _ = _one_call_e4m3(w, c8)
    rows = full_size_rows(w, seed=2)
    ref = oracle_attention_e4m3(w, c8, rows=rows, k_cache=torch.from_numpy(rk), v_cache=torch.from_numpy(rv))
    assert_parity(got, ref, w, rows=rows)
