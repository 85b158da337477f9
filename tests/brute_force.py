"""Pure-Python scalar brute force of the verify attention, used only to pin the oracle.

Written independently of ``oracle``: positions are classified one at a time, dot products and sums
use ``math.fsum`` and weights use ``math.exp``. Only for tiny shapes (a few thousand scalar ops).
"""
import math


def bf16_bits_to_float(u16):
    import struct
    return struct.unpack("<f", struct.pack("<I", (int(u16) & 0xFFFF) << 16))[0]


def fp16_bits_to_float(u16):
    import struct
    return struct.unpack("<e", struct.pack("<H", int(u16) & 0xFFFF))[0]


def brute_force_attention(q, k_cache, v_cache, block_tables, context_lens, num_candidates, masks,
                          scale, dtype):
    """Nested lists out[b][i][h][d] of Python floats. Inputs are uint16 bit arrays (numpy is fine)."""
    conv = bf16_bits_to_float if dtype == "bf16" else fp16_bits_to_float
    B, C, Hq, D = q.shape
    Hkv, bs = k_cache.shape[1], k_cache.shape[2]
    group = Hq // Hkv
    out = []
    for b in range(B):
        L = int(context_lens[b])
        n = int(num_candidates[b])
        first_candidate = L - n
        rows_b = []
        for i in range(C):
            heads = []
            for h in range(Hq):
                if i >= n:
                    heads.append([0.0] * D)
                    continue
                kvh = h // group
                qv = [conv(q[b, i, h, d]) for d in range(D)]
                logits, vals = [], []
                for p in range(L):
                    if p >= first_candidate:
                        j = p - first_candidate
                        if not ((int(masks[b][i]) >> j) & 1):
                            continue
                    blk = int(block_tables[b][p // bs])
                    slot = p % bs
                    kv = [conv(k_cache[blk, kvh, slot, d]) for d in range(D)]
                    logits.append(scale * math.fsum(qv[d] * kv[d] for d in range(D)))
                    vals.append([conv(v_cache[blk, kvh, slot, d]) for d in range(D)])
                if not logits:
                    heads.append([0.0] * D)
                    continue
                top = max(logits)
                w = [math.exp(s - top) for s in logits]
                tot = math.fsum(w)
                heads.append([math.fsum(w[k] * vals[k][d] for k in range(len(w))) / tot for d in range(D)])
            rows_b.append(heads)
        out.append(rows_b)
    return out
