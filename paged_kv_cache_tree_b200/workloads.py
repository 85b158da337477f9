"""Seeded synthetic inputs for paged tree-attention verify and paged KV-append.

This module only draws inputs; it holds none of the attention or append arithmetic, and it is the one
piece of code that both the CPU oracle's tests and the CUDA path's tests/bench share.

Shapes follow the workloads the TACO-LLM pages talk about: Llama-3.1-70B-like attention heads
(64 query / 8 KV heads, head_dim 128) verifying lookahead candidates, arranged as a chain or as a
forest-derived token tree, over a paged KV cache whose fixed-size blocks are reached through a block
table ("大模型倍速推理引擎 TACO-LLM 的设计与实践", 53ai.com workshop page, sections
"4. 支持 Paged Attention" and "优化方案设计思路"). The pages print no dataset; every value is
drawn here from a seeded CPU ``torch.Generator``.

Recipe (one generator per workload, seed = 1000 + k for the k-th named workload), in draw order:
  1. context lengths L_b (uniform integers, inclusive bounds; they count the candidates too);
  2. a random permutation of the physical block pool; sequence b takes the next ceil(L_b/bs) pool
     entries, in order, as its block table (unused table entries are -1);
  3. tree parents per sequence: a chain has parent[i] = i-1 (no draws); a forest draws parent[i]
     uniformly from {-1, 0, ..., i-1};
  4. q, then the K cache, then the V cache, then k_new, then v_new, all ~N(0,1) rounded to the dtype.
Pool size is ceil(1.1 * sum_b ceil(L_b/bs)) blocks unless a workload fixes it. Memory the verify must
never read (unmapped pool blocks, slots >= L_b of a sequence's last block, query rows of padding
candidates) is filled with NaN for parity runs (``fill="nan"``) or zeros for timed runs.

Candidate i of sequence b sits at logical position P_b + i with P_b = L_b - n_b. With
``candidates_in_cache=True`` the cache already holds k_new/v_new there (the state after a
paged KV-append); otherwise those slots are poisoned too and an append must fill them.

8-bit (e4m3) caches for a workload come from ``make_e4m3_cache``: byte patterns drawn directly (random
sign and mantissa, exponent field mostly in 9..14, sometimes anywhere in 0..14), the NaN code where the
16-bit caches hold NaN, and per-KV-head scales uniform on [0.004, 0.012]; no quantisation happens here.

Token streams for the prefix-tree lookup come from ``make_prefix_inputs`` (its docstring gives the
recipe); they hold token ids only, no hashing or matching. Token streams for the Lookahead Cache come
from ``make_lookahead_inputs`` (phrase-structured streams; its docstring gives the recipe).
"""
from __future__ import annotations

import dataclasses
import itertools
import math
from typing import Optional, Sequence, Union

import torch

# name -> spec; index k (1-based) gives the seed 1000 + k.
WORKLOADS = {
    "tiny": dict(k=1, dtype="fp16", B=2, Hq=4, Hkv=2, D=64, bs=16, C=4, tree="chain",
                 ctx=("fixed", [37, 100]), num_blocks=40),
    "decode": dict(k=2, dtype="bf16", B=64, Hq=32, Hkv=8, D=128, bs=16, C=1, tree="chain",
                   ctx=("uniform", 512, 4096)),
    "chain": dict(k=3, dtype="bf16", B=32, Hq=64, Hkv=8, D=128, bs=16, C=8, tree="chain",
                  ctx=("uniform", 1024, 8192)),
    "tree": dict(k=4, dtype="bf16", B=16, Hq=64, Hkv=8, D=128, bs=32, C=16, tree="forest",
                 ctx=("uniform", 2048, 16384)),
    "long": dict(k=5, dtype="bf16", B=4, Hq=64, Hkv=8, D=128, bs=64, C=4, tree="chain",
                 ctx=("uniform", 32768, 131072)),
}

WORKLOAD_DESCRIPTIONS = {
    "tiny": "tiny paged tree-attention: B2, 4q/2kv, D64, fp16, bs16, L={37,100}, 40 blocks, C=4 chain",
    "decode": "plain paged decode: B64, 32q/8kv, D128, bf16, bs16, L~U[512,4096], C=1",
    "chain": "lookahead chain verify: B32, 64q/8kv, D128, bf16, bs16, L~U[1024,8192], C=8 chain",
    "tree": "tree verify: B16, 64q/8kv, D128, bf16, bs32, L~U[2048,16384], C=16 random forest",
    "long": "long-sequence verify: B4, 64q/8kv, D128, bf16, bs64, L~U[32768,131072], C=4 chain",
}

TORCH_DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16}

_CHUNK = 1 << 24  # elements per randn call, so that huge caches are drawn without a giant fp32 temp


@dataclasses.dataclass
class Workload:
    """Host (CPU) tensors of one verify step. Shapes use B, C, Hq, Hkv, D, bs, NB, maxblk."""

    name: str
    dtype: str                    # "bf16" | "fp16"
    B: int
    C: int
    Hq: int
    Hkv: int
    D: int
    bs: int
    num_blocks: int
    max_blocks: int
    scale: float
    context_lens: torch.Tensor    # int32 [B]      L_b, candidates included
    num_candidates: torch.Tensor  # int32 [B]      n_b <= min(C, L_b)
    parents: torch.Tensor         # int32 [B, C]   parent index or -1
    tree_mask: torch.Tensor       # int32 [B, C]   uint32 bit pattern: bit j = row i may see candidate j
    block_tables: torch.Tensor    # int32 [B, maxblk], -1 where unmapped
    slot_offsets: torch.Tensor    # int32 [B, C]   P_b + i for i < n_b, else -1
    q: torch.Tensor               # [B, C, Hq, D]
    k_cache: torch.Tensor         # [NB, Hkv, bs, D]
    v_cache: torch.Tensor         # [NB, Hkv, bs, D]
    k_new: torch.Tensor           # [B, C, Hkv, D]
    v_new: torch.Tensor           # [B, C, Hkv, D]

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def kv_bytes(self) -> int:
        """K+V bytes the verify must read: sum_b L_b * Hkv * D * elt * 2."""
        return int(self.context_lens.long().sum()) * self.Hkv * self.D * 2 * 2

    def qo_bytes(self) -> int:
        """Q + O bytes: 2 * B * C * Hq * D * elt."""
        return 2 * self.B * self.C * self.Hq * self.D * 2

    def append_bytes(self) -> int:
        """K/V-append bytes moved: (read + write) of every appended row of K and V."""
        rows = int(self.num_candidates.long().sum())
        return 2 * 2 * rows * self.Hkv * self.D * 2

    def candidate_tokens(self) -> int:
        return int(self.num_candidates.long().sum())

    def to(self, device) -> "Workload":
        out = dataclasses.replace(self)
        for f in dataclasses.fields(self):
            v = getattr(self, f.name)
            if isinstance(v, torch.Tensor):
                setattr(out, f.name, v.to(device))
        return out


def _randn(n: int, g: torch.Generator, dtype: torch.dtype) -> torch.Tensor:
    out = torch.empty(n, dtype=dtype)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        out[s:e] = torch.randn(e - s, generator=g).to(dtype)
    return out


def chain_parents(C: int) -> list:
    return [i - 1 for i in range(C)]


def masks_from_parents(parents: Sequence[int], n: int) -> list:
    """Ancestor-or-self bit sets (bit j = candidate j) for rows i < n; rows i >= n get 0."""
    masks = []
    for i in range(len(parents)):
        if i >= n:
            masks.append(0)
            continue
        m = 1 << i
        p = parents[i]
        if p >= 0:
            m |= masks[p]
        masks.append(m)
    return masks


def _to_i32_bits(words: Sequence[int]) -> list:
    return [w - (1 << 32) if w >= (1 << 31) else w for w in words]


def make_workload(
    spec: Union[str, dict],
    *,
    seed: Optional[int] = None,
    fill: str = "nan",
    candidates_in_cache: bool = True,
    context_lens: Optional[Sequence[int]] = None,
    num_candidates: Optional[Sequence[int]] = None,
    parents: Optional[Sequence[Sequence[int]]] = None,
    pool_slack: float = 1.1,
    extra_table_cols: int = 0,
) -> Workload:
    """Draw one workload.

    ``spec`` is a name of ``WORKLOADS`` or a dict with the same keys (dtype, B, Hq, Hkv, D, bs, C,
    tree in {"chain", "forest"}, ctx = ("fixed", [..]) | ("uniform", lo, hi), optional num_blocks).
    ``context_lens`` / ``num_candidates`` / ``parents`` override what the spec would draw (the draws
    still happen, so the stream of later draws does not move).
    """
    if isinstance(spec, str):
        name = spec
        sp = dict(WORKLOADS[spec])
    else:
        sp = dict(spec)
        name = sp.get("name", "custom")
    if seed is None:
        seed = 1000 + int(sp.get("k", 0))
    if fill not in ("nan", "zero"):
        raise ValueError("fill must be 'nan' or 'zero'")
    tdt = TORCH_DTYPES[sp["dtype"]]
    B, C, Hq, Hkv, D, bs = (int(sp[x]) for x in ("B", "C", "Hq", "Hkv", "D", "bs"))
    g = torch.Generator().manual_seed(int(seed))

    # 1. context lengths
    ctx = sp["ctx"]
    if ctx[0] == "fixed":
        L = [int(x) for x in ctx[1]]
    else:
        L = [int(x) for x in torch.randint(int(ctx[1]), int(ctx[2]) + 1, (B,), generator=g)]
    if context_lens is not None:
        L = [int(x) for x in context_lens]
    assert len(L) == B
    if num_candidates is None:
        n = [min(C, Lb) for Lb in L]
    else:
        n = [int(x) for x in num_candidates]
    for b in range(B):
        if not (0 <= n[b] <= C and n[b] <= L[b]):
            raise ValueError(f"need 0 <= n_b <= min(C, L_b); got n={n[b]} L={L[b]} C={C}")

    # 2. block pool permutation and block tables
    nblk = [(Lb + bs - 1) // bs for Lb in L]
    total = sum(nblk)
    NB = int(sp.get("num_blocks") or math.ceil(pool_slack * total))
    NB = max(NB, total, 1)
    perm = torch.randperm(NB, generator=g)
    maxblk = max(max(nblk), 1) + int(extra_table_cols)
    bt = torch.full((B, maxblk), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        bt[b, : nblk[b]] = perm[off: off + nblk[b]].to(torch.int32)
        off += nblk[b]

    # 3. tree parents
    par = []
    for b in range(B):
        if sp["tree"] == "chain":
            pb = chain_parents(C)
        elif sp["tree"] == "forest":
            pb = [int(torch.randint(0, i + 1, (1,), generator=g)) - 1 for i in range(C)]
        else:
            raise ValueError("tree must be 'chain' or 'forest'")
        par.append(pb)
    if parents is not None:
        par = [list(map(int, p)) for p in parents]
    masks = [_to_i32_bits(masks_from_parents(par[b], n[b])) for b in range(B)]

    # 4. values
    q = _randn(B * C * Hq * D, g, tdt).view(B, C, Hq, D)
    k_cache = _randn(NB * Hkv * bs * D, g, tdt).view(NB, Hkv, bs, D)
    v_cache = _randn(NB * Hkv * bs * D, g, tdt).view(NB, Hkv, bs, D)
    k_new = _randn(B * C * Hkv * D, g, tdt).view(B, C, Hkv, D)
    v_new = _randn(B * C * Hkv * D, g, tdt).view(B, C, Hkv, D)

    poison = float("nan") if fill == "nan" else 0.0
    used = torch.zeros(NB, dtype=torch.bool)
    for b in range(B):
        blocks = bt[b, : nblk[b]].long()
        used[blocks] = True
        P = L[b] - n[b]
        if nblk[b] > 0:
            last = int(bt[b, nblk[b] - 1])
            tail = L[b] - (nblk[b] - 1) * bs          # valid slots in the last block
            k_cache[last, :, tail:, :] = poison
            v_cache[last, :, tail:, :] = poison
        for i in range(n[b]):
            p = P + i
            blk = int(bt[b, p // bs])
            if candidates_in_cache:
                k_cache[blk, :, p % bs, :] = k_new[b, i]
                v_cache[blk, :, p % bs, :] = v_new[b, i]
            else:
                k_cache[blk, :, p % bs, :] = poison
                v_cache[blk, :, p % bs, :] = poison
        q[b, n[b]:] = poison
        k_new[b, n[b]:] = poison
        v_new[b, n[b]:] = poison
    k_cache[~used] = poison
    v_cache[~used] = poison

    slots = torch.full((B, C), -1, dtype=torch.int32)
    for b in range(B):
        P = L[b] - n[b]
        for i in range(n[b]):
            slots[b, i] = P + i

    return Workload(
        name=name, dtype=sp["dtype"], B=B, C=C, Hq=Hq, Hkv=Hkv, D=D, bs=bs, num_blocks=NB,
        max_blocks=maxblk, scale=1.0 / math.sqrt(D),
        context_lens=torch.tensor(L, dtype=torch.int32),
        num_candidates=torch.tensor(n, dtype=torch.int32),
        parents=torch.tensor(par, dtype=torch.int32).view(B, C),
        tree_mask=torch.tensor(masks, dtype=torch.int32).view(B, C),
        block_tables=bt, slot_offsets=slots, q=q, k_cache=k_cache, v_cache=v_cache,
        k_new=k_new, v_new=v_new,
    )


@dataclasses.dataclass
class KV8Cache:
    """e4m3 caches of a workload: uint8 codes [NB, Hkv, bs, D] and float32 per-KV-head scales."""

    k_cache: torch.Tensor
    v_cache: torch.Tensor
    k_scale: torch.Tensor
    v_scale: torch.Tensor

    def to(self, device) -> "KV8Cache":
        return KV8Cache(*(getattr(self, f.name).to(device) for f in dataclasses.fields(self)))


E4M3_NAN = 0x7F


def _random_e4m3_codes(n: int, g: torch.Generator) -> torch.Tensor:
    """n random finite e4m3 byte patterns on the generator's device: sign and 3-bit mantissa uniform;
    the 4-bit exponent field uniform on 9..14 for 7 of 8 codes and on 0..14 (zeros and subnormals
    included) for the rest."""
    dev = g.device
    out = torch.empty(n, dtype=torch.uint8, device=dev)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        m = e - s
        draw = lambda lo, hi: torch.randint(lo, hi, (m,), generator=g, dtype=torch.int32, device=dev)
        sign, man, exp_hi, exp_all = draw(0, 2), draw(0, 8), draw(9, 15), draw(0, 15)
        wide = draw(0, 8) == 0
        ex = torch.where(wide, exp_all, exp_hi)
        out[s:e] = ((sign << 7) | (ex << 3) | man).to(torch.uint8)
    return out


def make_e4m3_cache(w: Workload, *, seed: Optional[int] = None) -> KV8Cache:
    """Seeded e4m3 caches with the block layout of ``w`` (drawn on the device ``w``'s caches live on):
    random finite codes wherever ``w``'s 16-bit caches hold numbers, the NaN code 0x7F wherever they hold
    NaN (unused blocks, slots past L_b and, unless the workload put them there, the candidates' slots);
    scales uniform on [0.004, 0.012]."""
    dev = w.k_cache.device
    g = torch.Generator(device=dev).manual_seed(int(seed if seed is not None else 77 + w.B * 131 + w.Hkv))
    shape = tuple(w.k_cache.shape)
    n = w.k_cache.numel()
    caches = []
    for src in (w.k_cache, w.v_cache):
        codes = _random_e4m3_codes(n, g).view(shape)
        codes[torch.isnan(src)] = E4M3_NAN
        caches.append(codes)
    k_scale = (0.004 + 0.008 * torch.rand(w.Hkv, generator=g, device=dev)).to(torch.float32)
    v_scale = (0.004 + 0.008 * torch.rand(w.Hkv, generator=g, device=dev)).to(torch.float32)
    return KV8Cache(caches[0], caches[1], k_scale, v_scale)


def kv8_attention_bytes(w: Workload) -> int:
    """Bytes the verify must move with e4m3 caches: K+V codes of every key, Q and O (16-bit)."""
    return int(w.context_lens.long().sum()) * w.Hkv * w.D * 2 + w.qo_bytes()


def kv8_append_bytes(w: Workload) -> int:
    """Quantising append: 16-bit rows read, e4m3 codes written, for K and V."""
    rows = int(w.num_candidates.long().sum())
    return 2 * rows * w.Hkv * w.D * (2 + 1)


@dataclasses.dataclass
class PrefixInputs:
    """Host tensors for the prefix-tree lookup: sequences whose KV blocks are cached (to insert) and the
    prompts of new requests (to look up)."""

    bs: int
    num_blocks: int
    max_blocks: int
    cached_tokens: torch.Tensor   # int32 [total]
    cached_starts: torch.Tensor   # int32 [S + 1]
    cached_tables: torch.Tensor   # int32 [S, max_blocks]: distinct physical blocks, -1 padded
    prompts: torch.Tensor         # int32 [total]
    prompt_starts: torch.Tensor   # int32 [B + 1]

    def seqs(self, which: str) -> list:
        toks = (self.cached_tokens if which == "cached" else self.prompts).tolist()
        st = (self.cached_starts if which == "cached" else self.prompt_starts).tolist()
        return [toks[st[i]:st[i + 1]] for i in range(len(st) - 1)]

    def prompt_tokens(self) -> int:
        return int(self.prompts.numel())

    def to(self, device) -> "PrefixInputs":
        out = dataclasses.replace(self)
        for f in dataclasses.fields(self):
            v = getattr(self, f.name)
            if isinstance(v, torch.Tensor):
                setattr(out, f.name, v.to(device))
        return out


def make_prefix_inputs(*, n_cached: int = 256, n_prompts: int = 64, bs: int = 16, n_stems: int = 8,
                       stem_len=(256, 2048), tail_len=(0, 4096), prompt_tail=(0, 2048), vocab: int = 128256,
                       seed: int = 2024) -> PrefixInputs:
    """Seeded token streams shaped like a serving cache: a few shared stems (system prompts); each
    cached sequence extends a stem or, half the time, a random-length prefix of an earlier cached
    sequence (so the cache forms a branching tree) with a random tail; each prompt is a random-length
    prefix of a cached sequence plus a divergent random tail (one in ten is wholly new). Tokens are
    uniform over the vocabulary; cached sequence i takes the next ceil(len/bs) entries of a random
    permutation of the block pool as its block table."""
    g = torch.Generator().manual_seed(int(seed))
    rint = lambda lo, hi: int(torch.randint(int(lo), int(hi) + 1, (1,), generator=g))
    rand_toks = lambda n: torch.randint(0, vocab, (n,), generator=g, dtype=torch.int32)
    stems = [rand_toks(rint(*stem_len)) for _ in range(n_stems)]
    cached = []
    for i in range(n_cached):
        if i > 0 and rint(0, 1) == 1:
            src = cached[rint(0, i - 1)]
            base = src[: rint(0, src.numel())]
        else:
            base = stems[rint(0, n_stems - 1)]
        cached.append(torch.cat([base, rand_toks(rint(*tail_len))]))
    prompts = []
    for _ in range(n_prompts):
        if rint(0, 9) == 0:
            prompts.append(rand_toks(rint(1, prompt_tail[1] + stem_len[1])))
        else:
            src = cached[rint(0, n_cached - 1)]
            prompts.append(torch.cat([src[: rint(0, src.numel())], rand_toks(rint(*prompt_tail))]))
    nblk = [(c.numel() + bs - 1) // bs for c in cached]
    max_blocks = max([1] + nblk + [(p.numel() + bs - 1) // bs for p in prompts])
    NB = max(1, math.ceil(1.1 * sum(nblk)))
    perm = torch.randperm(NB, generator=g).to(torch.int32)
    tables = torch.full((n_cached, max_blocks), -1, dtype=torch.int32)
    off = 0
    for i, k in enumerate(nblk):
        tables[i, :k] = perm[off:off + k]
        off += k
    starts = lambda seqs: torch.tensor([0] + list(itertools.accumulate(int(x.numel()) for x in seqs)), dtype=torch.int32)
    return PrefixInputs(bs=bs, num_blocks=NB, max_blocks=max_blocks, cached_tokens=torch.cat(cached),
                        cached_starts=starts(cached), cached_tables=tables, prompts=torch.cat(prompts),
                        prompt_starts=starts(prompts))


@dataclasses.dataclass
class LookaheadInputs:
    """Host tensors for the Lookahead Cache: each sequence's token history, a shared global token array
    (passages separated by -1) and per-sequence copy lengths."""

    history: torch.Tensor       # int32 [total]
    hist_starts: torch.Tensor   # int32 [B + 1]
    global_tokens: torch.Tensor  # int32 [G]
    copy_len: torch.Tensor      # int32 [B]
    max_match: int
    C: int

    def histories(self) -> list:
        h, st = self.history.tolist(), self.hist_starts.tolist()
        return [h[st[i]:st[i + 1]] for i in range(len(st) - 1)]

    def to(self, device) -> "LookaheadInputs":
        out = dataclasses.replace(self)
        for f in dataclasses.fields(self):
            v = getattr(self, f.name)
            if isinstance(v, torch.Tensor):
                setattr(out, f.name, v.to(device))
        return out


def _phrase_stream(g: torch.Generator, n: int, bank: list, vocab: int, p_phrase: float) -> torch.Tensor:
    parts, total = [], 0
    while total < n:
        if float(torch.rand(1, generator=g)) < p_phrase:
            part = bank[int(torch.randint(0, len(bank), (1,), generator=g))]
        else:
            part = torch.randint(0, vocab, (int(torch.randint(1, 9, (1,), generator=g)),), generator=g, dtype=torch.int32)
        parts.append(part)
        total += part.numel()
    return torch.cat(parts)[:n]


def make_lookahead_inputs(*, B: int = 64, hist_len=(512, 4096), n_docs: int = 16, doc_len=(1024, 4096),
                          n_phrases: int = 512, phrase_len=(2, 24), p_phrase: float = 0.8, vocab: int = 128256,
                          copy_len=(1, 8), max_match: int = 4, C: int = 16, seed: int = 4242) -> LookaheadInputs:
    """Seeded phrase-structured token streams (generated text repeats itself: the pages' premise). A bank
    of random phrases is drawn first; every stream concatenates phrases from the bank (with probability
    p_phrase) and short random runs. Sequence histories have lengths U[hist_len]; the global cache is
    n_docs streams of U[doc_len] tokens separated by -1; copy lengths are uniform in copy_len."""
    g = torch.Generator().manual_seed(int(seed))
    rint = lambda lo, hi: int(torch.randint(int(lo), int(hi) + 1, (1,), generator=g))
    bank = [torch.randint(0, vocab, (rint(*phrase_len),), generator=g, dtype=torch.int32) for _ in range(n_phrases)]
    hists = [_phrase_stream(g, rint(*hist_len), bank, vocab, p_phrase) for _ in range(B)]
    docs = []
    for _ in range(n_docs):
        docs += [_phrase_stream(g, rint(*doc_len), bank, vocab, p_phrase), torch.tensor([-1], dtype=torch.int32)]
    glob = torch.cat(docs) if docs else torch.zeros(0, dtype=torch.int32)
    cl = torch.randint(int(copy_len[0]), int(copy_len[1]) + 1, (B,), generator=g, dtype=torch.int32)
    starts = torch.tensor([0] + list(itertools.accumulate(int(h.numel()) for h in hists)), dtype=torch.int32)
    return LookaheadInputs(history=torch.cat(hists) if hists else torch.zeros(0, dtype=torch.int32),
                           hist_starts=starts, global_tokens=glob, copy_len=cl, max_match=max_match, C=C)


@dataclasses.dataclass
class AcceptInputs:
    """Host tensors of one acceptance step (after a verify): candidate tokens and target logits."""

    vocab: int
    tokens: torch.Tensor          # int32 [B, C]   candidate token ids (rows i >= n_b: -1)
    target_logits: torch.Tensor   # bf16/fp16 [B, C + 1, V]   row 0: after the prefix, row i + 1: after candidate i
    planted: torch.Tensor         # int32 [B, C + 1]  the index each row's margin was planted at

    def logits_bytes(self) -> int:
        return self.target_logits.numel() * self.target_logits.element_size()

    def to(self, device) -> "AcceptInputs":
        return AcceptInputs(self.vocab, self.tokens.to(device), self.target_logits.to(device), self.planted.to(device))


def make_accept_inputs(w: Workload, *, vocab: int = 128256, seed: Optional[int] = None, hit_prob: float = 0.7,
                       margin: float = 8.0, ties: bool = False) -> AcceptInputs:
    """Draw the target model's logits and the candidates' tokens for workload ``w``'s candidate trees.

    Recipe (one generator, seed = 5000 + the workload's seed unless given), in draw order:
      1. per (b, row) of the B x (C + 1) rows a planted index, uniform in [0, V);
      2. the logits, ~N(0, 1) rounded to ``w``'s dtype, then ``margin`` added at each planted index
         (so that row's largest value sits there; with ``ties`` every third row also gets the same
         value at a second, uniformly drawn index);
      3. per candidate a coin with P(hit) = ``hit_prob``: a hit copies the planted index of its
         parent's row (row 0 for a root), a miss draws a uniform index different from it.
    Vocabulary 128256 is the size of the Llama-3.1 tokenizer the pages' models use.
    """
    B, C = w.B, w.C
    if seed is None:
        seed = 5000 + int(w.context_lens.sum().item()) % 100000
    g = torch.Generator().manual_seed(int(seed))
    rows = C + 1
    planted = torch.randint(0, vocab, (B, rows), generator=g, dtype=torch.int64)
    logits = _randn(B * rows * vocab, g, TORCH_DTYPES[w.dtype]).view(B, rows, vocab)
    second = torch.randint(0, vocab, (B, rows), generator=g, dtype=torch.int64)
    for b in range(B):
        for r in range(rows):
            top = logits[b, r, planted[b, r]].float() + margin
            logits[b, r, planted[b, r]] = top
            if ties and (b * rows + r) % 3 == 0 and int(second[b, r]) != int(planted[b, r]):
                logits[b, r, second[b, r]] = logits[b, r, planted[b, r]]
    coins = torch.rand((B, C), generator=g)
    other = torch.randint(0, vocab - 1, (B, C), generator=g, dtype=torch.int64)
    tokens = torch.full((B, C), -1, dtype=torch.int32)
    for b in range(B):
        for i in range(int(w.num_candidates[b])):
            p = int(w.parents[b, i])
            want = int(planted[b, 0 if p < 0 else p + 1])
            if float(coins[b, i]) < hit_prob:
                tokens[b, i] = want
            else:
                o = int(other[b, i])
                tokens[b, i] = o if o < want else o + 1
    return AcceptInputs(vocab=vocab, tokens=tokens, target_logits=logits, planted=planted.to(torch.int32))


def to_numpy_bits(t: torch.Tensor):
    """Raw 16-bit patterns of a bf16/fp16 tensor as a numpy uint16 array (no value conversion)."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")


def as_uint32(t: torch.Tensor):
    """int32 tensor holding uint32 bit patterns -> numpy uint32 array."""
    return t.contiguous().numpy().view("uint32")
