"""CPU oracle for paged tree-attention verify and paged KV-append.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module. The product path (the CUDA library and its Python binding)
never calls it, and this module imports nothing from the product.

What it computes is the plain definition, in float64, written out slowly and directly:

* Paging ("大模型倍速推理引擎 TACO-LLM 的设计与实践", 53ai.com workshop page, section
  "4. 支持 Paged Attention"): each sequence's KV cache is cut into blocks holding a fixed number of
  tokens, and consecutive logical blocks map to non-contiguous physical blocks through a block table.
  Logical position p of sequence b therefore lives in physical block ``block_tables[b][p // bs]`` at
  slot ``p % bs``.
* Verification (same page, sections "TACO-LLM 如何解决大模型推理瓶颈?" and "优化方案设计思路"): the
  target model checks several candidate tokens in one forward pass, so each sequence brings n_b query
  rows (the candidates), which sit at the last n_b logical positions P_b .. L_b - 1 (P_b = L_b - n_b).
* Tree attention (same page, section "优化策略总结", item 1): candidates that share a prefix share its
  computation; each candidate attends to the committed prefix and to its own ancestors only. Bit j of
  ``tree_mask_bits[b][i]`` says candidate row i may see candidate j (bits j >= n_b are ignored).
* Flash-style fusion and split-KV (the TurboAttention bullets under "整体方案分为两大部分"; and the
  TurboAttention section of the 618zxw.cn article) are exact re-associations of the softmax, so the
  oracle evaluates the softmax in one piece.

Open points the pages leave and the reading taken here:
* GQA: query head h reads KV head h // (Hq / Hkv).
* ``scale`` multiplies the logits before the softmax.
* Rows i >= n_b of the output, and rows whose visible set is empty, are exact zeros.

Every function here is pinned by tests against closed forms, library routines and brute force
(block-permutation invariance, one-key context, equal keys, scale 0, chain mask == causal attention,
ancestor-only dependence, a pure-Python brute force); none is "parity unpinned".
"""
from __future__ import annotations

import numpy as np


def widen_to_f64(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of 16-bit float patterns (uint16) to float64.

    bf16 is the upper half of an IEEE binary32, so shifting the pattern left by 16 bits gives the
    binary32 with the same value; fp16 is IEEE binary16, which numpy reads natively. Both widen to
    float64 without rounding.
    """
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == "bf16":
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    if dtype == "fp16":
        return bits.view(np.float16).astype(np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")


def gather_sequence_kv(cache: np.ndarray, table_row: np.ndarray, kv_head: int, length: int,
                       block_size: int) -> np.ndarray:
    """K (or V) rows of logical positions 0 .. length-1 of one sequence and one KV head.

    ``cache`` is [num_blocks, Hkv, block_size, D] (any dtype); positions are walked one by one through
    the block table: position p -> block table_row[p // block_size], slot p % block_size.
    """
    D = cache.shape[-1]
    out = np.empty((length, D), dtype=cache.dtype)
    for p in range(length):
        phys = int(table_row[p // block_size])
        out[p] = cache[phys, kv_head, p % block_size]
    return out


def visible_positions(length: int, n_cand: int, row: int, mask_word: int) -> np.ndarray:
    """Logical key positions candidate ``row`` may attend to.

    The committed prefix 0 .. P-1 (P = length - n_cand) is always visible; candidate j (at position
    P + j, j < n_cand) is visible iff bit j of ``mask_word`` is set. Positions >= length never are.
    """
    P = length - n_cand
    vis = list(range(P))
    for j in range(n_cand):
        if (int(mask_word) >> j) & 1:
            vis.append(P + j)
    return np.asarray(vis, dtype=np.int64)


def softmax_attend(q_row: np.ndarray, keys: np.ndarray, values: np.ndarray, visible: np.ndarray,
                   scale: float) -> np.ndarray:
    """sum over visible p of softmax(scale * q.k_p) v_p, in float64; zeros if nothing is visible.

    ``keys``/``values`` hold every position of the sequence; ``visible`` is a boolean vector over the
    same positions. Invisible positions take no part: their logits and values are never used.
    """
    if not visible.any():
        return np.zeros(values.shape[-1], dtype=np.float64)
    s = scale * (keys @ q_row)
    s = s[visible]
    w = np.exp(s - s.max())
    return (w @ values[visible]) / w.sum()


def _widen_kv(x: np.ndarray, kv_dtype: str, scale, g: int) -> np.ndarray:
    """K or V rows of KV head g as float64: 16-bit floats widen exactly; e4m3 codes decode and take
    the head's scale (see ``oracle.fp8``)."""
    if kv_dtype == "e4m3":
        from .fp8 import e4m3_decode

        return e4m3_decode(x) * float(np.asarray(scale, dtype=np.float64)[g])
    return widen_to_f64(x, kv_dtype)


def paged_tree_attention(q, k_cache, v_cache, block_tables, context_lens, num_candidates,
                         tree_mask_bits, scale, dtype, rows=None, kv_dtype=None, k_scale=None, v_scale=None):
    """Oracle of the verify attention.

    q: uint16 bits [B, C, Hq, D]; k_cache, v_cache: uint16 bits [NB, Hkv, bs, D] (or uint8 e4m3
    codes with ``kv_dtype="e4m3"`` and per-KV-head float scales ``k_scale`` / ``v_scale``);
    block_tables: int [B, maxblk]; context_lens, num_candidates: int [B];
    tree_mask_bits: uint32 [B, C]; dtype: "bf16" | "fp16" (of q, and of K/V unless kv_dtype is given).
    rows: optional iterable of (b, i, h) to evaluate; other rows are left as NaN.
    Returns float64 [B, C, Hq, D] (not rounded to the storage dtype).
    """
    kvd = dtype if kv_dtype is None else kv_dtype
    B, C, Hq, D = q.shape
    Hkv, bs = k_cache.shape[1], k_cache.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, C, Hq, D), dtype=np.float64)
    want = None
    if rows is not None:
        out[:] = np.nan
        want = {}
        for (b, i, h) in rows:
            want.setdefault((int(b), int(h) // G), []).append((int(i), int(h)))
    for b in range(B):
        L = int(context_lens[b])
        n = int(num_candidates[b])
        for g in range(Hkv):
            if want is not None and (b, g) not in want:
                continue
            K = _widen_kv(gather_sequence_kv(k_cache, block_tables[b], g, L, bs), kvd, k_scale, g)
            V = _widen_kv(gather_sequence_kv(v_cache, block_tables[b], g, L, bs), kvd, v_scale, g)
            pairs = want[(b, g)] if want is not None else [(i, h) for i in range(C)
                                                              for h in range(g * G, (g + 1) * G)]
            for (i, h) in pairs:
                if i >= n:
                    out[b, i, h] = 0.0
                    continue
                visible = np.zeros(L, dtype=bool)
                visible[visible_positions(L, n, i, int(tree_mask_bits[b][i]))] = True
                qh = widen_to_f64(q[b, i, h], dtype)
                out[b, i, h] = softmax_attend(qh, K, V, visible, float(scale))
    return out


def paged_kv_append(k_new, v_new, block_tables, slot_offsets, k_cache, v_cache):
    """Oracle of the KV-append: returns new (k_cache, v_cache) with the candidates' rows copied in.

    For each (b, i) with s = slot_offsets[b][i] >= 0 and each KV head h, the 16-bit patterns of
    k_new[b, i, h, :] are copied to k_cache[block_tables[b][s // bs], h, s % bs, :] (same for V);
    every other byte stays as it was. Inputs are uint16 bit arrays; nothing is converted.
    """
    kc = np.array(k_cache, copy=True)
    vc = np.array(v_cache, copy=True)
    B, C, Hkv, D = k_new.shape
    bs = kc.shape[2]
    for b in range(B):
        for i in range(C):
            s = int(slot_offsets[b][i])
            if s < 0:
                continue
            phys = int(block_tables[b][s // bs])
            for h in range(Hkv):
                kc[phys, h, s % bs, :] = k_new[b, i, h, :]
                vc[phys, h, s % bs, :] = v_new[b, i, h, :]
    return kc, vc


def within_tolerance(gpu: np.ndarray, ref: np.ndarray, atol: float = 1e-2, rtol: float = 2e-2) -> np.ndarray:
    """Elementwise acceptance |gpu - ref| <= atol + rtol * |ref| (NaN never passes)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return np.abs(gpu - ref) <= atol + rtol * np.abs(ref)
