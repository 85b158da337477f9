"""CPU oracle for an 8-bit (e4m3) paged KV cache with per-KV-head scales.

TEST INFRASTRUCTURE ONLY (imported by ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline leg, never by the product path).

The pages ("大模型倍速推理引擎 TACO-LLM 的设计与实践" and its companion article) list quantised
attention operators among the engine's kernels but fix no format. The reading taken here:

* e4m3 is the 8-bit float with 1 sign, 4 exponent (bias 7) and 3 mantissa bits, no infinities,
  0x7F / 0xFF are NaN, the largest finite magnitude is 448 (S.1111.110), subnormals are
  m * 2^-9 (m = 1..7).
* A cache entry is stored as e4m3(float32(x) / float32(scale[h])) for KV head h: the quotient is the
  correctly rounded float32 division, and the conversion rounds to the nearest e4m3 value (ties to
  the even mantissa), saturating magnitudes above 448 to 448; NaN stays NaN.
* Reading an entry gives decode(byte) * scale[h], exactly (float64).

Pinned by tests: every one of the 254 finite codes round-trips; encoding equals a brute-force search
over all codes for the nearest value; ties go to the even code; saturation and signed zeros.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """float64 values of e4m3 byte codes (NaN for 0x7F / 0xFF)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = sign * (1.0 + m / 8.0) * np.exp2(e - 7.0)
    sub = sign * (m / 8.0) * 2.0 ** -6
    v = np.where(e == 0, sub, normal)
    return np.where((c & 0x7F) == 0x7F, np.nan, v)


_FINITE_CODES = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
_FINITE_VALUES = e4m3_decode(_FINITE_CODES)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Nearest e4m3 code of each float (ties to the even mantissa), saturating at +-448, NaN -> 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint8)
    flat_x = x.reshape(-1)
    flat_o = out.reshape(-1)
    # non-negative codes 0x00..0x7E in increasing value order
    pos_codes = np.arange(0x7F, dtype=np.uint8)
    pos_vals = e4m3_decode(pos_codes)
    for k, v in enumerate(flat_x):
        if np.isnan(v):
            flat_o[k] = 0x7F
            continue
        a = min(abs(v), E4M3_MAX)
        j = int(np.searchsorted(pos_vals, a))  # first value >= a
        if j < len(pos_vals) and pos_vals[j] == a:
            c = j
        else:
            lo, hi = j - 1, j
            dlo, dhi = a - pos_vals[lo], pos_vals[hi] - a
            if dlo < dhi:
                c = lo
            elif dhi < dlo:
                c = hi
            else:
                c = lo if (lo & 1) == 0 else hi  # tie: the even mantissa
        code = int(pos_codes[c])
        if np.signbit(v):
            code |= 0x80
        flat_o[k] = code
    return out


def quantize_rows(rows_bits: np.ndarray, dtype: str, scale: np.ndarray) -> np.ndarray:
    """e4m3 codes of 16-bit float rows [..., Hkv, D] divided (float32) by scale[Hkv]."""
    from .paged_attention import widen_to_f64

    x32 = widen_to_f64(rows_bits, dtype).astype(np.float32)
    s32 = np.asarray(scale, dtype=np.float32)[:, None]
    q = (x32 / s32).astype(np.float32)
    return e4m3_encode(q.astype(np.float64))


def paged_kv_append_e4m3(k_new_bits, v_new_bits, dtype, block_tables, slot_offsets, k_scale, v_scale,
                         k_cache, v_cache):
    """Quantised paged append: returns new (k_cache, v_cache) uint8 arrays [NB, Hkv, bs, D]."""
    k_cache = np.array(k_cache, copy=True)
    v_cache = np.array(v_cache, copy=True)
    B, C = slot_offsets.shape
    bs = k_cache.shape[2]
    for b in range(B):
        for i in range(C):
            s = int(slot_offsets[b, i])
            if s < 0:
                continue
            blk = int(block_tables[b, s // bs])
            k_cache[blk, :, s % bs, :] = quantize_rows(k_new_bits[b, i], dtype, k_scale)
            v_cache[blk, :, s % bs, :] = quantize_rows(v_new_bits[b, i], dtype, v_scale)
    return k_cache, v_cache


def dequantize_cache(cache_codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """float64 [NB, Hkv, bs, D] values of an e4m3 cache with per-head scales."""
    return e4m3_decode(cache_codes) * np.asarray(scale, dtype=np.float64)[None, :, None, None]
