"""ctypes binding of libtaco_attn (argument marshalling only).

Every function here takes torch tensors for device memory and a CUDA stream, turns them into the
pointers and sizes of the C ABI in ``include/taco_attn.h`` and calls it. No arithmetic of the method
happens here, and there is no fallback: if the shared library is missing or a call fails, an
exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtaco_attn.so")

TACO_OK = 0
TACO_ERR_INVALID_ARG = 1
TACO_ERR_UNSUPPORTED = 2
TACO_ERR_CUDA = 3
TACO_ERR_DEVICE_CHECK = 4

TACO_DTYPE_F16 = 0
TACO_DTYPE_BF16 = 1

TACO_OPT_GRID_CTAS = 1
TACO_OPT_KERNEL = 2
TACO_OPT_L2_PREFETCH = 3
TACO_OPT_TEST_STALL = 4
TACO_OPT_SEG_COST = 5
TACO_OPT_COMBINE = 6

EXPORTED = (
    "paged_tree_attention",
    "paged_kv_append",
    "paged_tree_attention_noalloc",
    "paged_tree_attention_append",
    "paged_tree_attention_e4m3",
    "paged_tree_attention_append_e4m3",
    "paged_kv_append_e4m3",
    "taco_attn_last_error",
    "taco_attn_check_device",
    "taco_attn_check_noalloc",
    "taco_attn_release_workspace",
    "taco_attn_set_option",
    "taco_attn_version",
    "taco_attn_last_call_launches",
    "tree_mask_from_parents",
    "logits_argmax",
    "tree_greedy_accept",
    "prefix_cache_lookup",
    "prefix_cache_insert",
    "lookahead_propose",
    "lookahead_update_copy_len",
)

_lib = None


class TacoError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"libtaco_attn status {status}: {message}")
        self.status = status


def load() -> ctypes.CDLL:
    """Load the in-tree library (built by ``paged_kv_cache_tree_b200.build_lib``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_tree_b200.build_lib`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    lib.paged_tree_attention.argtypes = [vp] * 7 + [f32, vp] + [i32] * 9 + [vp]
    lib.paged_tree_attention.restype = i32
    lib.paged_tree_attention_noalloc.argtypes = [vp] * 7 + [f32, vp] + [i32] * 9 + [vp]
    lib.paged_tree_attention_noalloc.restype = i32
    lib.paged_tree_attention_append.argtypes = [vp] * 9 + [f32, vp] + [i32] * 9 + [vp]
    lib.paged_tree_attention_append.restype = i32
    lib.paged_kv_append.argtypes = [vp] * 6 + [i32] * 8 + [vp]
    lib.paged_kv_append.restype = i32
    lib.paged_tree_attention_e4m3.argtypes = [vp] * 9 + [f32, vp] + [i32] * 9 + [vp]
    lib.paged_tree_attention_e4m3.restype = i32
    lib.paged_tree_attention_append_e4m3.argtypes = [vp] * 11 + [f32, vp] + [i32] * 9 + [vp]
    lib.paged_tree_attention_append_e4m3.restype = i32
    lib.paged_kv_append_e4m3.argtypes = [vp] * 8 + [i32] * 8 + [vp]
    lib.paged_kv_append_e4m3.restype = i32
    lib.taco_attn_last_error.argtypes = []
    lib.taco_attn_last_error.restype = ctypes.c_char_p
    lib.taco_attn_check_device.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.taco_attn_check_device.restype = i32
    lib.taco_attn_check_noalloc.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.taco_attn_check_noalloc.restype = i32
    lib.taco_attn_release_workspace.argtypes = []
    lib.taco_attn_release_workspace.restype = None
    lib.taco_attn_set_option.argtypes = [i32, ctypes.c_int64]
    lib.taco_attn_set_option.restype = i32
    lib.taco_attn_version.argtypes = []
    lib.taco_attn_version.restype = i32
    lib.taco_attn_last_call_launches.argtypes = []
    lib.taco_attn_last_call_launches.restype = i32
    lib.tree_mask_from_parents.argtypes = [vp, vp, i32, i32, vp, vp]
    lib.tree_mask_from_parents.restype = i32
    lib.logits_argmax.argtypes = [vp, i32, ctypes.c_int64, i32, vp, vp]
    lib.logits_argmax.restype = i32
    lib.tree_greedy_accept.argtypes = [vp] * 5 + [i32, i32] + [vp] * 4 + [vp]
    lib.tree_greedy_accept.restype = i32
    i64 = ctypes.c_int64
    lib.prefix_cache_lookup.argtypes = [vp] * 4 + [i64] + [vp] * 5 + [i32] * 4 + [vp]
    lib.prefix_cache_lookup.restype = i32
    lib.prefix_cache_insert.argtypes = [vp] * 5 + [i64] + [vp] * 5 + [i32] * 4 + [vp]
    lib.prefix_cache_insert.restype = i32
    lib.lookahead_propose.argtypes = [vp] * 3 + [i64, vp, i32, i32, i32] + [vp] * 3 + [vp]
    lib.lookahead_propose.restype = i32
    lib.lookahead_update_copy_len.argtypes = [vp] * 4 + [i32, i32, f32, i32, vp]
    lib.lookahead_update_copy_len.restype = i32
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != TACO_OK:
        msg = load().taco_attn_last_error().decode(errors="replace")
        raise TacoError(status, msg)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return TACO_DTYPE_BF16
    if t.dtype == torch.float16:
        return TACO_DTYPE_F16
    raise TypeError(f"unsupported dtype {t.dtype}; expected bfloat16 or float16")


def _stream_handle(stream: Optional[torch.cuda.Stream], device: torch.device) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return int(s.cuda_stream)


def _need_cuda(name: str, t: torch.Tensor, dtype=None, ndim=None) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got {t.dim()}")


def paged_tree_attention(q, k_cache, v_cache, block_tables, context_lens, num_candidates, tree_mask_bits,
                         scale: float, out: Optional[torch.Tensor] = None, stream=None,
                         _entry: str = "paged_tree_attention") -> torch.Tensor:
    """q [B,C,Hq,D]; k/v_cache [NB,Hkv,bs,D]; block_tables int32 [B,maxblk]; context_lens and
    num_candidates int32 [B]; tree_mask_bits int32/uint32 [B,C] (bit patterns). Returns ``out``."""
    _need_cuda("q", q, (torch.bfloat16, torch.float16), 4)
    _need_cuda("k_cache", k_cache, q.dtype, 4)
    _need_cuda("v_cache", v_cache, q.dtype, 4)
    _need_cuda("block_tables", block_tables, torch.int32, 2)
    _need_cuda("context_lens", context_lens, torch.int32, 1)
    _need_cuda("num_candidates", num_candidates, torch.int32, 1)
    _need_cuda("tree_mask_bits", tree_mask_bits, (torch.int32, torch.uint32), 2)
    B, C, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("k_cache / v_cache shape mismatch with q")
    if block_tables.shape[0] != B or context_lens.shape[0] != B or num_candidates.shape[0] != B:
        raise ValueError("batch dimension mismatch")
    if tuple(tree_mask_bits.shape) != (B, C):
        raise ValueError("tree_mask_bits must be [B, C]")
    if out is None:
        out = torch.empty_like(q)
    _need_cuda("out", out, q.dtype, 4)
    if tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must have q's shape")
    lib = load()
    _check(getattr(lib, _entry)(
        q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_tables.data_ptr(), context_lens.data_ptr(),
        num_candidates.data_ptr(), tree_mask_bits.data_ptr(), float(scale), out.data_ptr(),
        _dtype_code(q), B, C, Hq, Hkv, D, bs, NB, block_tables.shape[1],
        _stream_handle(stream, q.device)))
    return out


def paged_tree_attention_noalloc(q, k_cache, v_cache, block_tables, context_lens, num_candidates,
                                 tree_mask_bits, scale: float, out: Optional[torch.Tensor] = None,
                                 stream=None) -> torch.Tensor:
    """Same as paged_tree_attention, through the entry point that allocates no device memory (its
    scratch is a fixed 24 MiB array in the library; see include/taco_attn.h for its limits)."""
    return paged_tree_attention(q, k_cache, v_cache, block_tables, context_lens, num_candidates, tree_mask_bits,
                                scale, out=out, stream=stream, _entry="paged_tree_attention_noalloc")


def paged_tree_attention_append(q, k_new, v_new, k_cache, v_cache, block_tables, context_lens, num_candidates,
                                tree_mask_bits, scale: float, out: Optional[torch.Tensor] = None,
                                stream=None) -> torch.Tensor:
    """Append the candidates' K/V (k_new, v_new [B,C,Hkv,D]) at slots P_b + i, then attend; returns out."""
    _need_cuda("q", q, (torch.bfloat16, torch.float16), 4)
    _need_cuda("k_new", k_new, q.dtype, 4)
    _need_cuda("v_new", v_new, q.dtype, 4)
    _need_cuda("k_cache", k_cache, q.dtype, 4)
    _need_cuda("v_cache", v_cache, q.dtype, 4)
    B, C, Hq, D = q.shape
    if tuple(k_new.shape) != (B, C, k_cache.shape[1], D) or tuple(v_new.shape) != tuple(k_new.shape):
        raise ValueError("k_new / v_new must be [B, C, Hkv, D]")
    if out is None:
        out = torch.empty_like(q)
    _need_cuda("block_tables", block_tables, torch.int32, 2)
    _need_cuda("context_lens", context_lens, torch.int32, 1)
    _need_cuda("num_candidates", num_candidates, torch.int32, 1)
    _need_cuda("tree_mask_bits", tree_mask_bits, (torch.int32, torch.uint32), 2)
    _need_cuda("out", out, q.dtype, 4)
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("shape mismatch")
    if block_tables.shape[0] != B or context_lens.shape[0] != B or num_candidates.shape[0] != B:
        raise ValueError("batch dimension mismatch")
    if tuple(tree_mask_bits.shape) != (B, C):
        raise ValueError("tree_mask_bits must be [B, C]")
    _check(load().paged_tree_attention_append(
        q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
        block_tables.data_ptr(), context_lens.data_ptr(), num_candidates.data_ptr(), tree_mask_bits.data_ptr(),
        float(scale), out.data_ptr(), _dtype_code(q), B, C, Hq, Hkv, D, bs, NB, block_tables.shape[1],
        _stream_handle(stream, q.device)))
    return out


def paged_kv_append(k_new, v_new, block_tables, slot_offsets, k_cache, v_cache, stream=None) -> None:
    """k_new, v_new [B,C,Hkv,D]; slot_offsets int32 [B,C] (-1 = skip); caches updated in place."""
    _need_cuda("k_new", k_new, (torch.bfloat16, torch.float16), 4)
    _need_cuda("v_new", v_new, k_new.dtype, 4)
    _need_cuda("block_tables", block_tables, torch.int32, 2)
    _need_cuda("slot_offsets", slot_offsets, torch.int32, 2)
    _need_cuda("k_cache", k_cache, k_new.dtype, 4)
    _need_cuda("v_cache", v_cache, k_new.dtype, 4)
    B, C, Hkv, D = k_new.shape
    NB, Hkv2, bs, D2 = k_cache.shape
    if (Hkv2, D2) != (Hkv, D) or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(v_new.shape) != tuple(k_new.shape):
        raise ValueError("shape mismatch between new rows and caches")
    if tuple(slot_offsets.shape) != (B, C) or block_tables.shape[0] != B:
        raise ValueError("slot_offsets must be [B, C] and block_tables [B, maxblk]")
    lib = load()
    _check(lib.paged_kv_append(
        k_new.data_ptr(), v_new.data_ptr(), block_tables.data_ptr(), slot_offsets.data_ptr(),
        k_cache.data_ptr(), v_cache.data_ptr(), _dtype_code(k_new), B, C, Hkv, D, bs, NB,
        block_tables.shape[1], _stream_handle(stream, k_new.device)))


def _need_scales(k_scale, v_scale, Hkv: int) -> None:
    for name, t in (("k_scale", k_scale), ("v_scale", v_scale)):
        _need_cuda(name, t, torch.float32, 1)
        if t.shape[0] != Hkv:
            raise ValueError(f"{name} must be float32 [num_kv_heads]")


def paged_tree_attention_e4m3(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, num_candidates,
                              tree_mask_bits, scale: float, out: Optional[torch.Tensor] = None,
                              stream=None, k_new=None, v_new=None) -> torch.Tensor:
    """Attention over e4m3 caches: q [B,C,Hq,D] bf16/fp16; k/v_cache uint8 [NB,Hkv,bs,D] e4m3 codes;
    k_scale / v_scale float32 [Hkv] (value = decode(code) * scale[h]). Returns ``out`` (q's dtype).
    With ``k_new`` / ``v_new`` ([B,C,Hkv,D], q's dtype) the candidates are first appended (quantised)
    at slots P_b .. L_b - 1 in the same call (paged_tree_attention_append_e4m3)."""
    _need_cuda("q", q, (torch.bfloat16, torch.float16), 4)
    _need_cuda("k_cache", k_cache, torch.uint8, 4)
    _need_cuda("v_cache", v_cache, torch.uint8, 4)
    _need_cuda("block_tables", block_tables, torch.int32, 2)
    _need_cuda("context_lens", context_lens, torch.int32, 1)
    _need_cuda("num_candidates", num_candidates, torch.int32, 1)
    _need_cuda("tree_mask_bits", tree_mask_bits, (torch.int32, torch.uint32), 2)
    B, C, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("k_cache / v_cache shape mismatch with q")
    if block_tables.shape[0] != B or context_lens.shape[0] != B or num_candidates.shape[0] != B:
        raise ValueError("batch dimension mismatch")
    if tuple(tree_mask_bits.shape) != (B, C):
        raise ValueError("tree_mask_bits must be [B, C]")
    _need_scales(k_scale, v_scale, Hkv)
    if out is None:
        out = torch.empty_like(q)
    _need_cuda("out", out, q.dtype, 4)
    if tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must have q's shape")
    if k_new is not None or v_new is not None:
        for name, t in (("k_new", k_new), ("v_new", v_new)):
            _need_cuda(name, t, q.dtype, 4)
            if tuple(t.shape) != (B, C, Hkv, D):
                raise ValueError(f"{name} must be [B, C, Hkv, D]")
        _check(load().paged_tree_attention_append_e4m3(
            q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
            k_scale.data_ptr(), v_scale.data_ptr(), block_tables.data_ptr(), context_lens.data_ptr(),
            num_candidates.data_ptr(), tree_mask_bits.data_ptr(), float(scale), out.data_ptr(), _dtype_code(q), B, C,
            Hq, Hkv, D, bs, NB, block_tables.shape[1], _stream_handle(stream, q.device)))
        return out
    _check(load().paged_tree_attention_e4m3(
        q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), k_scale.data_ptr(), v_scale.data_ptr(),
        block_tables.data_ptr(), context_lens.data_ptr(), num_candidates.data_ptr(), tree_mask_bits.data_ptr(),
        float(scale), out.data_ptr(), _dtype_code(q), B, C, Hq, Hkv, D, bs, NB, block_tables.shape[1],
        _stream_handle(stream, q.device)))
    return out


def paged_kv_append_e4m3(k_new, v_new, block_tables, slot_offsets, k_scale, v_scale, k_cache, v_cache,
                         stream=None) -> None:
    """Quantising append: k_new, v_new [B,C,Hkv,D] bf16/fp16; k/v_cache uint8 [NB,Hkv,bs,D] e4m3 codes,
    updated in place with e4m3(x / scale[h]); slot_offsets int32 [B,C] (-1 = skip)."""
    _need_cuda("k_new", k_new, (torch.bfloat16, torch.float16), 4)
    _need_cuda("v_new", v_new, k_new.dtype, 4)
    _need_cuda("block_tables", block_tables, torch.int32, 2)
    _need_cuda("slot_offsets", slot_offsets, torch.int32, 2)
    _need_cuda("k_cache", k_cache, torch.uint8, 4)
    _need_cuda("v_cache", v_cache, torch.uint8, 4)
    B, C, Hkv, D = k_new.shape
    NB, Hkv2, bs, D2 = k_cache.shape
    if (Hkv2, D2) != (Hkv, D) or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(v_new.shape) != tuple(k_new.shape):
        raise ValueError("shape mismatch between new rows and caches")
    if tuple(slot_offsets.shape) != (B, C) or block_tables.shape[0] != B:
        raise ValueError("slot_offsets must be [B, C] and block_tables [B, maxblk]")
    _need_scales(k_scale, v_scale, Hkv)
    _check(load().paged_kv_append_e4m3(
        k_new.data_ptr(), v_new.data_ptr(), block_tables.data_ptr(), slot_offsets.data_ptr(), k_scale.data_ptr(),
        v_scale.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), _dtype_code(k_new), B, C, Hkv, D, bs, NB,
        block_tables.shape[1], _stream_handle(stream, k_new.device)))


def tree_mask_from_parents(parents, num_candidates, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """parents int32 [B, C] (-1 = root); num_candidates int32 [B]. Returns uint32 bit patterns in an
    int32 [B, C] tensor (the tree_mask_bits of paged_tree_attention)."""
    _need_cuda("parents", parents, torch.int32, 2)
    _need_cuda("num_candidates", num_candidates, torch.int32, 1)
    B, C = parents.shape
    if num_candidates.shape[0] != B:
        raise ValueError("batch dimension mismatch")
    if out is None:
        out = torch.empty_like(parents)
    _need_cuda("out", out, (torch.int32, torch.uint32), 2)
    if tuple(out.shape) != (B, C):
        raise ValueError("out must be [B, C]")
    _check(load().tree_mask_from_parents(parents.data_ptr(), num_candidates.data_ptr(), B, C, out.data_ptr(),
                                         _stream_handle(stream, parents.device)))
    return out


def logits_argmax(logits, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """logits [..., V] bf16/fp16 (dense). Returns int32 [...]: per row the smallest index of the largest
    value (NaN never wins; a row without a number above -inf gives 0)."""
    _need_cuda("logits", logits, (torch.bfloat16, torch.float16))
    V = logits.shape[-1]
    rows = logits.numel() // V if V > 0 else 0
    if out is None:
        out = torch.empty(logits.shape[:-1], dtype=torch.int32, device=logits.device)
    _need_cuda("out", out, torch.int32)
    if out.numel() != rows:
        raise ValueError("out must have one entry per row")
    _check(load().logits_argmax(logits.data_ptr(), _dtype_code(logits), rows, V, out.data_ptr(),
                                _stream_handle(stream, logits.device)))
    return out


def tree_greedy_accept(target_argmax, candidate_tokens, parents, num_candidates, context_lens, stream=None):
    """target_argmax int32 [B, C+1]; candidate_tokens, parents int32 [B, C]; num_candidates, context_lens
    int32 [B]. Returns (accept_len [B], accepted_path [B, C], bonus_token [B], slot_offsets [B, C])."""
    _need_cuda("target_argmax", target_argmax, torch.int32, 2)
    _need_cuda("candidate_tokens", candidate_tokens, torch.int32, 2)
    _need_cuda("parents", parents, torch.int32, 2)
    _need_cuda("num_candidates", num_candidates, torch.int32, 1)
    _need_cuda("context_lens", context_lens, torch.int32, 1)
    B, C = candidate_tokens.shape
    if tuple(parents.shape) != (B, C) or tuple(target_argmax.shape) != (B, C + 1):
        raise ValueError("parents must be [B, C] and target_argmax [B, C + 1]")
    if num_candidates.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("batch dimension mismatch")
    dev = candidate_tokens.device
    accept_len = torch.empty(B, dtype=torch.int32, device=dev)
    path = torch.empty(B, C, dtype=torch.int32, device=dev)
    bonus = torch.empty(B, dtype=torch.int32, device=dev)
    slots = torch.empty(B, C, dtype=torch.int32, device=dev)
    _check(load().tree_greedy_accept(
        target_argmax.data_ptr(), candidate_tokens.data_ptr(), parents.data_ptr(), num_candidates.data_ptr(),
        context_lens.data_ptr(), B, C, accept_len.data_ptr(), path.data_ptr(), bonus.data_ptr(), slots.data_ptr(),
        _stream_handle(stream, dev)))
    return accept_len, path, bonus, slots


def check_device(stream=None, device=None) -> int:
    """Synchronise the stream and return the device error bits (raises TacoError if any are set)."""
    lib = load()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    bits = ctypes.c_uint32(0)
    st = lib.taco_attn_check_device(_stream_handle(stream, dev), ctypes.byref(bits))
    _check(st)
    return int(bits.value)


def check_noalloc(stream=None, device=None) -> int:
    """Synchronise the stream and return the error bits of paged_tree_attention_noalloc's fixed scratch
    (raises TacoError if any are set); the word is cleared."""
    lib = load()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    bits = ctypes.c_uint32(0)
    st = lib.taco_attn_check_noalloc(_stream_handle(stream, dev), ctypes.byref(bits))
    _check(st)
    return int(bits.value)


def set_option(key: int, value: int) -> None:
    _check(load().taco_attn_set_option(int(key), int(value)))


def release_workspace() -> None:
    load().taco_attn_release_workspace()


def version() -> int:
    return int(load().taco_attn_version())


def last_call_launches() -> int:
    """Kernels the calling thread's last attention call enqueued (see include/taco_attn.h)."""
    return int(load().taco_attn_last_call_launches())


class PrefixCache:
    """Device memory of a prefix tree of full KV blocks (see prefix_cache_* in include/taco_attn.h):
    an open-addressing slot table and per-physical-block node arrays, allocated and initialised here
    with torch (plumbing only); lookups and inserts run in the library's kernels."""

    def __init__(self, num_blocks: int, block_size: int, capacity: int, device="cuda"):
        if capacity < 2 or capacity & (capacity - 1):
            raise ValueError("capacity must be a power of two >= 2")
        self.num_blocks, self.block_size, self.capacity = int(num_blocks), int(block_size), int(capacity)
        self.slot_keys = torch.zeros(capacity, dtype=torch.int64, device=device)     # uint64 bit patterns
        self.slot_nodes = torch.full((capacity,), -1, dtype=torch.int32, device=device)
        self.node_parent = torch.full((num_blocks,), -1, dtype=torch.int32, device=device)
        self.node_depth = torch.full((num_blocks,), -1, dtype=torch.int32, device=device)
        self.node_tokens = torch.zeros((num_blocks, block_size), dtype=torch.int32, device=device)

    @staticmethod
    def _check_seqs(tokens, seq_starts):
        _need_cuda("tokens", tokens, torch.int32, 1)
        _need_cuda("seq_starts", seq_starts, torch.int32, 1)
        if seq_starts.shape[0] < 1:
            raise ValueError("seq_starts must hold batch + 1 offsets")
        if tokens.numel() == 0:   # the C ABI wants a real pointer even when no token is read
            tokens = torch.zeros(1, dtype=torch.int32, device=tokens.device)
        return seq_starts.shape[0] - 1, tokens

    def lookup(self, tokens, seq_starts, max_blocks: int, out_blocks=None, out_matched=None, stream=None):
        """Longest cached run of each sequence's leading full blocks: (out_blocks [B, max_blocks]
        physical blocks then -1, out_matched [B] blocks matched)."""
        B, tokens = self._check_seqs(tokens, seq_starts)
        if out_blocks is None:
            out_blocks = torch.empty((B, max_blocks), dtype=torch.int32, device=tokens.device)
        if out_matched is None:
            out_matched = torch.empty((B,), dtype=torch.int32, device=tokens.device)
        _need_cuda("out_blocks", out_blocks, torch.int32, 2)
        _need_cuda("out_matched", out_matched, torch.int32, 1)
        if tuple(out_blocks.shape) != (B, max_blocks) or out_matched.shape[0] != B:
            raise ValueError("out_blocks must be [B, max_blocks] and out_matched [B]")
        _check(load().prefix_cache_lookup(
            tokens.data_ptr(), seq_starts.data_ptr(), self.slot_keys.data_ptr(), self.slot_nodes.data_ptr(),
            self.capacity, self.node_parent.data_ptr(), self.node_depth.data_ptr(), self.node_tokens.data_ptr(),
            out_blocks.data_ptr(), out_matched.data_ptr(), B, self.block_size, self.num_blocks, max_blocks,
            _stream_handle(stream, tokens.device)))
        return out_blocks, out_matched

    def insert(self, tokens, seq_starts, block_tables, out_blocks=None, out_inserted=None, stream=None):
        """Insert each sequence's full blocks (K/V in block_tables [B, max_blocks]); returns
        (out_blocks [B, max_blocks]: the block holding each prefix afterwards, then -1; out_inserted [B])."""
        B, tokens = self._check_seqs(tokens, seq_starts)
        _need_cuda("block_tables", block_tables, torch.int32, 2)
        if block_tables.shape[0] != B:
            raise ValueError("block_tables must be [B, max_blocks]")
        max_blocks = block_tables.shape[1]
        if out_blocks is None:
            out_blocks = torch.empty((B, max_blocks), dtype=torch.int32, device=tokens.device)
        if out_inserted is None:
            out_inserted = torch.empty((B,), dtype=torch.int32, device=tokens.device)
        _need_cuda("out_blocks", out_blocks, torch.int32, 2)
        _need_cuda("out_inserted", out_inserted, torch.int32, 1)
        _check(load().prefix_cache_insert(
            tokens.data_ptr(), seq_starts.data_ptr(), block_tables.data_ptr(), self.slot_keys.data_ptr(),
            self.slot_nodes.data_ptr(), self.capacity, self.node_parent.data_ptr(), self.node_depth.data_ptr(),
            self.node_tokens.data_ptr(), out_blocks.data_ptr(), out_inserted.data_ptr(), B, self.block_size,
            self.num_blocks, max_blocks, _stream_handle(stream, tokens.device)))
        return out_blocks, out_inserted


def lookahead_propose(history, hist_starts, global_tokens, copy_len, max_match: int, max_candidates: int,
                      stream=None):
    """Candidate forests (tokens [B, C], parents [B, C], num_candidates [B]) from each sequence's history
    (int32 tokens, hist_starts [B + 1]) and a shared global token array (int32, may be empty)."""
    _need_cuda("history", history, torch.int32, 1)
    _need_cuda("hist_starts", hist_starts, torch.int32, 1)
    _need_cuda("global_tokens", global_tokens, torch.int32, 1)
    _need_cuda("copy_len", copy_len, torch.int32, 1)
    B = hist_starts.shape[0] - 1
    if B < 0 or copy_len.shape[0] != B:
        raise ValueError("hist_starts must be [B + 1] and copy_len [B]")
    if history.numel() == 0:
        history = torch.zeros(1, dtype=torch.int32, device=history.device)
    dev = history.device
    tok = torch.empty((B, max_candidates), dtype=torch.int32, device=dev)
    par = torch.empty((B, max_candidates), dtype=torch.int32, device=dev)
    num = torch.empty((B,), dtype=torch.int32, device=dev)
    g_ptr = global_tokens.data_ptr() if global_tokens.numel() > 0 else None
    _check(load().lookahead_propose(history.data_ptr(), hist_starts.data_ptr(), g_ptr, global_tokens.numel(),
                                    copy_len.data_ptr(), max_match, B, max_candidates, tok.data_ptr(), par.data_ptr(),
                                    num.data_ptr(), _stream_handle(stream, dev)))
    return tok, par, num


def lookahead_update_copy_len(accept_len, num_proposed, hit, copy_len, copy_max: int, alpha: float = 0.5,
                              batch_ref: int = 16, stream=None) -> None:
    """Updates hit (float32 [B]) and copy_len (int32 [B]) in place from a verify step's accept lengths."""
    _need_cuda("accept_len", accept_len, torch.int32, 1)
    _need_cuda("num_proposed", num_proposed, torch.int32, 1)
    _need_cuda("hit", hit, torch.float32, 1)
    _need_cuda("copy_len", copy_len, torch.int32, 1)
    B = accept_len.shape[0]
    if num_proposed.shape[0] != B or hit.shape[0] != B or copy_len.shape[0] != B:
        raise ValueError("all arrays must be [B]")
    _check(load().lookahead_update_copy_len(accept_len.data_ptr(), num_proposed.data_ptr(), hit.data_ptr(),
                                            copy_len.data_ptr(), B, copy_max, float(alpha), batch_ref,
                                            _stream_handle(stream, accept_len.device)))
