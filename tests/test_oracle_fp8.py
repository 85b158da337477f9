"""Pins of the e4m3 KV-cache oracle (oracle/fp8.py): exhaustive round trips, a brute-force nearest-value
search, hand-worked ties and saturation, and agreement with the 16-bit oracle on exactly representable
values."""
import math

import numpy as np
import pytest

import oracle
from oracle import fp8


def brute_encode(v: float) -> int:
    """Nearest finite code by scanning all of them; ties to the even code; beyond 448 saturates."""
    if math.isnan(v):
        return 0x7F
    a = min(abs(v), 448.0)
    best, bd = None, None
    for c in range(0x7F):                      # non-negative finite codes
        d = abs(fp8.e4m3_decode(np.array([c]))[0] - a)
        if bd is None or d < bd or (d == bd and (c & 1) == 0 and (best & 1) == 1):
            best, bd = c, d
    return best | (0x80 if math.copysign(1.0, v) < 0 else 0)


def test_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = fp8.e4m3_decode(codes)
    assert np.array_equal(fp8.e4m3_encode(vals), codes)
    assert np.isnan(fp8.e4m3_decode(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def test_encode_matches_a_brute_force_search():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.normal(0, 1, 300), rng.normal(0, 100, 100), rng.uniform(-2e-3, 2e-3, 100),
                        rng.uniform(440, 600, 20), -rng.uniform(440, 600, 20)])
    got = fp8.e4m3_encode(x)
    assert [int(c) for c in got] == [brute_encode(float(v)) for v in x]


@pytest.mark.parametrize("v,code", [
    (1.0, 0x38), (448.0, 0x7E), (-448.0, 0xFE), (1000.0, 0x7E), (2.0 ** -9, 0x01), (2.0 ** -10, 0x00),
    (3 * 2.0 ** -10, 0x02), (1.0625, 0x38), (1.1875, 0x3A), (-0.0, 0x80), (0.0, 0x00), (7 * 2.0 ** -9, 0x07),
    (15 * 2.0 ** -10, 0x08), (464.0, 0x7E),
])
def test_hand_worked_values(v, code):
    assert int(fp8.e4m3_encode(np.array([v]))[0]) == code


def test_quantised_attention_equals_16_bit_attention_on_representable_values():
    """With scale 1 and K/V that are e4m3 values (all exact in bf16) both oracles see the same numbers."""
    rng = np.random.default_rng(1)
    B, C, Hq, Hkv, D, bs, NB = 2, 3, 4, 2, 8, 4, 12
    kcodes = rng.integers(0, 256, (NB, Hkv, bs, D)).astype(np.uint8)
    vcodes = rng.integers(0, 256, (NB, Hkv, bs, D)).astype(np.uint8)
    kcodes[(kcodes & 0x7F) == 0x7F] = 0x38
    vcodes[(vcodes & 0x7F) == 0x7F] = 0x38
    to_bf16 = lambda v: (np.asarray(v, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    kb, vb = to_bf16(fp8.e4m3_decode(kcodes)), to_bf16(fp8.e4m3_decode(vcodes))
    assert np.array_equal(oracle.widen_to_f64(kb, "bf16"), fp8.e4m3_decode(kcodes))
    q = to_bf16(rng.normal(0, 0.05, (B, C, Hq, D)))
    bt = np.arange(12, dtype=np.int32).reshape(2, 6)
    ctx, nc = np.array([17, 9]), np.array([3, 2])
    masks = np.array([[1, 3, 7], [1, 2, 0]], dtype=np.uint32)
    ones = np.ones(Hkv)
    a = oracle.paged_tree_attention(q, kcodes, vcodes, bt, ctx, nc, masks, 0.3, "bf16", kv_dtype="e4m3",
                                    k_scale=ones, v_scale=ones)
    b = oracle.paged_tree_attention(q, kb, vb, bt, ctx, nc, masks, 0.3, "bf16")
    assert np.array_equal(a, b)
    # a scale multiplies the values the attention sees
    c = oracle.paged_tree_attention(q, kcodes, vcodes, bt, ctx, nc, masks, 0.3, "bf16", kv_dtype="e4m3",
                                    k_scale=ones, v_scale=2 * ones)
    assert np.allclose(c, 2 * a, rtol=0, atol=0)


def test_quantised_append_writes_only_the_slots():
    rng = np.random.default_rng(2)
    B, C, Hkv, D, bs, NB = 2, 3, 2, 8, 4, 6
    kn = (rng.normal(0, 3, (B, C, Hkv, D)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    vn = (rng.normal(0, 3, (B, C, Hkv, D)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    kc = rng.integers(0, 256, (NB, Hkv, bs, D)).astype(np.uint8)
    vc = kc.copy()
    bt = np.array([[3, 1, -1], [0, 5, 2]], dtype=np.int32)
    so = np.array([[5, 6, -1], [9, -1, 1]], dtype=np.int32)
    ks, vs = np.array([0.5, 2.0]), np.array([1.0, 0.25])
    k2, v2 = fp8.paged_kv_append_e4m3(kn, vn, "bf16", bt, so, ks, vs, kc, vc)
    touched = np.zeros((NB, bs), dtype=bool)
    for b in range(B):
        for i in range(C):
            s = so[b, i]
            if s < 0:
                continue
            blk = bt[b, s // bs]
            touched[blk, s % bs] = True
            x = oracle.widen_to_f64(kn[b, i], "bf16").astype(np.float32) / np.float32(ks)[:, None]
            assert np.array_equal(k2[blk, :, s % bs], fp8.e4m3_encode(x.astype(np.float64)))
    for blk in range(NB):
        for sl in range(bs):
            if not touched[blk, sl]:
                assert np.array_equal(k2[blk, :, sl], kc[blk, :, sl])


def test_nan_encodes_to_the_positive_nan_code_and_both_nan_codes_decode_to_nan():
    # the reading: NaN stays NaN, as 0x7F whatever its sign; 0x7F and 0xFF are e4m3's only NaN codes
    codes = fp8.e4m3_encode(np.array([np.nan, -np.nan, np.float64("nan")]))
    assert codes.tolist() == [0x7F, 0x7F, 0x7F]
    vals = fp8.e4m3_decode(np.array([0x7F, 0xFF, 0x7E, 0xFE], dtype=np.uint8))
    assert np.isnan(vals[0]) and np.isnan(vals[1]) and vals[2] == 448.0 and vals[3] == -448.0
