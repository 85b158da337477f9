"""The allocation-free verify entry point against the regular one (needs a B200).

paged_tree_attention_noalloc serves callers that cannot allocate device memory (a fixed memory-pool
budget, no implicit synchronisation mid-step, no allocation after start-up): it takes its split-KV
scratch from a fixed array inside the library instead of cudaMalloc. This file is collected last so
that a run stopping at its first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_tree_b200 as taco
from paged_kv_cache_tree_b200 import _lib
from paged_kv_cache_tree_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _call(entry, d, w, out):
    lib = _lib.load()
    B, C, Hq, D = d.q.shape
    NB, Hkv, bs, _ = d.k_cache.shape
    status = getattr(lib, entry)(
        d.q.data_ptr(), d.k_cache.data_ptr(), d.v_cache.data_ptr(), d.block_tables.data_ptr(),
        d.context_lens.data_ptr(), d.num_candidates.data_ptr(), d.tree_mask.data_ptr(), ctypes.c_float(w.scale),
        out.data_ptr(), _lib.TACO_DTYPE_BF16 if d.q.dtype == torch.bfloat16 else _lib.TACO_DTYPE_F16,
        B, C, Hq, Hkv, D, bs, NB, d.block_tables.shape[1], torch.cuda.current_stream().cuda_stream)
    assert status == _lib.TACO_OK, lib.taco_attn_last_error()


@pytest.mark.parametrize("spec", [
    dict(dtype="bf16", B=8, Hq=32, Hkv=8, D=128, bs=16, C=4, tree="forest", ctx=("uniform", 200, 3000)),
    dict(dtype="fp16", B=4, Hq=64, Hkv=8, D=128, bs=32, C=8, tree="chain", ctx=("uniform", 100, 2500)),
])
def test_noalloc_matches_regular_entry_point_twice(spec):
    torch.cuda.set_device(0)
    w = wl.make_workload(spec, seed=77)
    d = w.to("cuda")
    ref = torch.empty_like(d.q)
    _call("paged_tree_attention", d, w, ref)
    torch.cuda.synchronize()
    ref_f = oracle.widen_to_f64(wl.to_numpy_bits(ref.cpu()), w.dtype)
    for _ in range(2):                                   # the scratch keeps the last call's contents
        got = torch.full_like(d.q, float("nan"))
        _call("paged_tree_attention_noalloc", d, w, got)
        torch.cuda.synchronize()
        got_f = oracle.widen_to_f64(wl.to_numpy_bits(got.cpu()), w.dtype)
        ok = oracle.within_tolerance(got_f, ref_f, 1e-2, 2e-2)
        assert ok.all(), f"max |diff| {np.nanmax(np.abs(got_f - ref_f))}"


def test_noalloc_rejects_calls_beyond_its_scratch():
    lib = _lib.load()
    # 70000 sequences * 1 KV head = 70000 work units > 65536: rejected on the host, nothing enqueued
    status = lib.paged_tree_attention_noalloc(16, 16, 16, 16, 16, 16, 16, ctypes.c_float(0.1), 16, 1, 70000, 1, 1, 1,
                                              128, 16, 100, 10, None)
    assert status == _lib.TACO_ERR_UNSUPPORTED
    assert "scratch" in lib.taco_attn_last_error().decode()
