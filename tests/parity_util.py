"""Helpers shared by the GPU parity tests: run one verify step through the C ABI and through the
oracle on the same seeded inputs, and compare them."""
import numpy as np
import torch

import oracle
import paged_kv_cache_tree_b200 as taco
from paged_kv_cache_tree_b200 import workloads as wl

ATOL = 1e-2
RTOL = 2e-2


def gpu_step(w, device="cuda", append=True):
    """Append (optional) then attention on the GPU; returns (out, k_cache, v_cache) on the host."""
    d = w.to(device)
    if append:
        taco.paged_kv_append(d.k_new, d.v_new, d.block_tables, d.slot_offsets, d.k_cache, d.v_cache)
    out = torch.full_like(d.q, float("nan"))
    taco.paged_tree_attention(d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, d.num_candidates,
                              d.tree_mask, w.scale, out=out)
    bits = taco.check_device()
    assert bits == 0
    return out.cpu(), d.k_cache, d.v_cache


def full_size_rows(w, seed, extra=24):
    """Rows (b, i, h) for a full-size parity check: one of every (sequence, KV head) unit (a random live
    candidate and a random head of the group), so that every unit and every split piece is merged and
    checked, plus `extra` random rows and the first and last row."""
    rng = np.random.default_rng(seed)
    G = w.Hq // w.Hkv
    rows = {(0, 0, 0), (w.B - 1, max(0, int(w.num_candidates[-1]) - 1), w.Hq - 1)}
    for b in range(w.B):
        n = max(1, int(w.num_candidates[b]))
        for g in range(w.Hkv):
            rows.add((b, int(rng.integers(n)), g * G + int(rng.integers(G))))
    for _ in range(extra):
        b = int(rng.integers(w.B))
        rows.add((b, int(rng.integers(max(1, int(w.num_candidates[b])))), int(rng.integers(w.Hq))))
    return sorted(rows)


def oracle_inputs(w):
    return dict(q=wl.to_numpy_bits(w.q), k_cache=wl.to_numpy_bits(w.k_cache), v_cache=wl.to_numpy_bits(w.v_cache),
                block_tables=w.block_tables.numpy(), context_lens=w.context_lens.numpy(),
                num_candidates=w.num_candidates.numpy(), tree_mask_bits=wl.as_uint32(w.tree_mask),
                scale=w.scale, dtype=w.dtype)


def oracle_step(w, append=True, rows=None):
    a = oracle_inputs(w)
    if append:
        a["k_cache"], a["v_cache"] = oracle.paged_kv_append(
            wl.to_numpy_bits(w.k_new), wl.to_numpy_bits(w.v_new), a["block_tables"], w.slot_offsets.numpy(),
            a["k_cache"], a["v_cache"])
    return oracle.paged_tree_attention(**a, rows=rows), a["k_cache"], a["v_cache"]


def as_f64(t: torch.Tensor, dtype: str) -> np.ndarray:
    return oracle.widen_to_f64(wl.to_numpy_bits(t), dtype)


def assert_parity(gpu_out: torch.Tensor, ref: np.ndarray, w, rows=None):
    """Rows i < n_b within |gpu - ref| <= ATOL + RTOL |ref|; rows i >= n_b exact +0 bit patterns."""
    got = as_f64(gpu_out, w.dtype)
    bits = wl.to_numpy_bits(gpu_out)
    n = w.num_candidates.numpy()
    if rows is None:
        rows = [(b, i, h) for b in range(w.B) for i in range(w.C) for h in range(w.Hq)]
    bad = []
    worst = 0.0
    for (b, i, h) in rows:
        if i >= n[b]:
            if np.any(bits[b, i, h] != 0):
                bad.append((b, i, h, "padding row not +0"))
            continue
        ok = oracle.within_tolerance(got[b, i, h], ref[b, i, h], ATOL, RTOL)
        err = np.abs(got[b, i, h] - ref[b, i, h])
        worst = max(worst, float(np.nanmax(err)) if np.isfinite(err).all() else float("inf"))
        if not ok.all():
            bad.append((b, i, h, float(np.max(err))))
    assert not bad, f"{len(bad)} rows out of tolerance, first: {bad[:5]}; worst |err| {worst}"
    return worst
