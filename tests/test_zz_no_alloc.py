"""The allocation-free verify entry point (needs a B200).

paged_tree_attention_noalloc serves callers that cannot allocate device memory: a server whose memory
pool already owns all free HBM, code that must not take cudaMalloc's implicit device synchronisation in
the middle of a step, and hosts that forbid allocation after start-up. It takes its split-KV scratch
from a fixed array inside the library instead of cudaMalloc. Every call is made through the C ABI and
compared with the CPU oracle, with the regular entry point, and with itself on a second call (the array
keeps the last call's contents, so the second call must not depend on them). This file is collected
last so that a run stopping at its first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_tree_b200 as taco
from paged_kv_cache_tree_b200 import _lib
from paged_kv_cache_tree_b200 import workloads as wl
from tests.parity_util import ATOL, RTOL, assert_parity, oracle_step

pytestmark = pytest.mark.gpu


def _call(entry, d, w, out, block_tables=None):
    lib = _lib.load()
    B, C, Hq, D = d.q.shape
    NB, Hkv, bs, _ = d.k_cache.shape
    bt = d.block_tables if block_tables is None else block_tables
    status = getattr(lib, entry)(
        d.q.data_ptr(), d.k_cache.data_ptr(), d.v_cache.data_ptr(), bt.data_ptr(),
        d.context_lens.data_ptr(), d.num_candidates.data_ptr(), d.tree_mask.data_ptr(), ctypes.c_float(w.scale),
        out.data_ptr(), _lib.TACO_DTYPE_BF16 if d.q.dtype == torch.bfloat16 else _lib.TACO_DTYPE_F16,
        B, C, Hq, Hkv, D, bs, NB, bt.shape[1], torch.cuda.current_stream().cuda_stream)
    assert status == _lib.TACO_OK, lib.taco_attn_last_error()


def _noalloc_bits():
    lib = _lib.load()
    bits = ctypes.c_uint32(0)
    st = lib.taco_attn_check_noalloc(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), ctypes.byref(bits))
    return st, int(bits.value)


SPECS = [
    # 16 packed rows, short contexts: the mma.sync kernel
    dict(dtype="bf16", B=8, Hq=32, Hkv=8, D=128, bs=16, C=4, tree="forest", ctx=("uniform", 200, 3000)),
    # 64 packed rows (a chain verify): the tcgen05 kernel, as in paged_tree_attention
    dict(dtype="fp16", B=4, Hq=64, Hkv=8, D=128, bs=32, C=8, tree="chain", ctx=("uniform", 100, 2500)),
    # few long sequences: every unit is split over several CTAs, so the log-sum-exp merge reads
    # 128-row partials from the fixed array
    dict(dtype="bf16", B=2, Hq=64, Hkv=8, D=128, bs=32, C=8, tree="forest", ctx=("uniform", 6000, 9000)),
    # 128 packed rows (a tree verify) on the tcgen05 kernel
    dict(dtype="bf16", B=3, Hq=64, Hkv=8, D=128, bs=32, C=16, tree="forest", ctx=("uniform", 500, 4000)),
    # 32 packed rows, long contexts: mma.sync with split units merged through the fixed array
    dict(dtype="bf16", B=2, Hq=64, Hkv=8, D=128, bs=64, C=4, tree="chain", ctx=("uniform", 5000, 9000)),
    # head_dim 64 on the tcgen05 kernel
    dict(dtype="bf16", B=3, Hq=32, Hkv=4, D=64, bs=16, C=8, tree="forest", ctx=("uniform", 300, 2000)),
]


@pytest.mark.parametrize("spec", SPECS)
def test_noalloc_matches_oracle_and_regular_entry_point_twice(spec):
    torch.cuda.set_device(0)
    w = wl.make_workload(spec, seed=77)
    d = w.to("cuda")
    want, _, _ = oracle_step(w, append=False)
    ref = torch.full_like(d.q, float("nan"))
    _call("paged_tree_attention", d, w, ref)
    torch.cuda.synchronize()
    assert taco.check_device() == 0
    ref_f = oracle.widen_to_f64(wl.to_numpy_bits(ref.cpu()), w.dtype)
    runs = []
    for _ in range(2):                                   # the scratch keeps the last call's contents
        got = torch.full_like(d.q, float("nan"))
        _call("paged_tree_attention_noalloc", d, w, got)
        torch.cuda.synchronize()
        assert _noalloc_bits() == (_lib.TACO_OK, 0)
        assert_parity(got.cpu(), want, w)                # against the oracle, element by element
        got_f = oracle.widen_to_f64(wl.to_numpy_bits(got.cpu()), w.dtype)
        ok = oracle.within_tolerance(got_f, ref_f, ATOL, RTOL)
        assert ok.all(), f"max |diff| vs regular entry point {np.nanmax(np.abs(got_f - ref_f))}"
        runs.append(wl.to_numpy_bits(got.cpu()))
    assert np.array_equal(runs[0], runs[1]), "two noalloc calls on the same inputs differ"


def test_noalloc_reports_a_bad_block_id_through_its_own_error_word():
    torch.cuda.set_device(0)
    spec = dict(dtype="bf16", B=2, Hq=8, Hkv=2, D=128, bs=16, C=2, tree="chain", ctx=("fixed", [40, 70]))
    w = wl.make_workload(spec, seed=2)
    d = w.to("cuda")
    bt = d.block_tables.clone()
    bt[1, 2] = w.num_blocks + 5                          # a mapped entry pointing past the pool
    out = torch.empty_like(d.q)
    assert _noalloc_bits() == (_lib.TACO_OK, 0)
    _call("paged_tree_attention_noalloc", d, w, out, block_tables=bt)
    # a second, clean call must not clear the first call's bit
    _call("paged_tree_attention_noalloc", d, w, out)
    torch.cuda.synchronize()
    assert taco.check_device() == 0                      # the regular word never sees it
    with pytest.raises(taco.TacoError) as ei:
        taco.check_noalloc()
    assert "block id" in str(ei.value)
    assert _noalloc_bits() == (_lib.TACO_OK, 0)          # read and cleared
    want, _, _ = oracle_step(w, append=False)
    _call("paged_tree_attention_noalloc", d, w, out)
    assert_parity(out.cpu(), want, w)
    assert _noalloc_bits() == (_lib.TACO_OK, 0)


def test_noalloc_rejects_calls_beyond_its_scratch():
    lib = _lib.load()
    # 70000 sequences * 1 KV head = 70000 work units > 65536: rejected on the host, nothing enqueued
    status = lib.paged_tree_attention_noalloc(16, 16, 16, 16, 16, 16, 16, ctypes.c_float(0.1), 16, 1, 70000, 1, 1, 1,
                                              128, 16, 100, 10, None)
    assert status == _lib.TACO_ERR_UNSUPPORTED
    assert "scratch" in lib.taco_attn_last_error().decode()
