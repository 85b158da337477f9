"""The C-ABI library loads without a GPU, exports every symbol its header declares, and rejects bad
arguments on the host before touching CUDA (CPU only)."""
import ctypes
import os
import re

import pytest

from paged_kv_cache_tree_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "taco_attn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", text)) - {"defined", "if", "sizeof"})


@pytest.fixture(scope="module")
def lib():
    return _lib.load()


def test_header_declares_the_boundary():
    names = declared_functions()
    assert "paged_tree_attention" in names and "paged_kv_append" in names
    assert set(names) == set(_lib.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.taco_attn_version() == 8


def _attn_args(**over):
    a = dict(q=16, k=16, v=16, bt=16, ctx=16, nc=16, mask=16, scale=0.125, out=16, dtype=1, B=2, C=4,
             Hq=8, Hkv=2, D=128, bs=16, NB=40, maxblk=8, stream=None)
    a.update(over)
    return [a["q"], a["k"], a["v"], a["bt"], a["ctx"], a["nc"], a["mask"], ctypes.c_float(a["scale"]), a["out"],
            a["dtype"], a["B"], a["C"], a["Hq"], a["Hkv"], a["D"], a["bs"], a["NB"], a["maxblk"], a["stream"]]


@pytest.mark.parametrize("over,status", [
    (dict(q=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(out=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(mask=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(dtype=7), _lib.TACO_ERR_INVALID_ARG),
    (dict(D=96), _lib.TACO_ERR_UNSUPPORTED),
    (dict(bs=24), _lib.TACO_ERR_UNSUPPORTED),
    (dict(bs=4), _lib.TACO_ERR_UNSUPPORTED),
    (dict(C=33), _lib.TACO_ERR_UNSUPPORTED),
    (dict(C=0), _lib.TACO_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), _lib.TACO_ERR_INVALID_ARG),
    (dict(B=-1), _lib.TACO_ERR_INVALID_ARG),
    (dict(NB=0), _lib.TACO_ERR_INVALID_ARG),
    (dict(maxblk=0), _lib.TACO_ERR_INVALID_ARG),
    (dict(q=24), _lib.TACO_ERR_INVALID_ARG),        # not 16-byte aligned
    (dict(scale=float("nan")), _lib.TACO_ERR_INVALID_ARG),
])
def test_attention_rejects_bad_arguments_on_host(lib, over, status):
    assert lib.paged_tree_attention(*_attn_args(**over)) == status
    assert lib.taco_attn_last_error().decode()


def test_attention_empty_batch_is_a_no_op(lib):
    assert lib.paged_tree_attention(*_attn_args(B=0)) == _lib.TACO_OK


@pytest.mark.parametrize("over,status", [
    (dict(kn=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(so=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(D=32), _lib.TACO_ERR_UNSUPPORTED),
    (dict(bs=1000), _lib.TACO_ERR_UNSUPPORTED),
    (dict(kc=8), _lib.TACO_ERR_INVALID_ARG),
])
def test_append_rejects_bad_arguments_on_host(lib, over, status):
    a = dict(kn=16, vn=16, bt=16, so=16, kc=16, vc=16, dtype=0, B=2, C=4, Hkv=2, D=64, bs=16, NB=40,
             maxblk=8, stream=None)
    a.update(over)
    args = [a["kn"], a["vn"], a["bt"], a["so"], a["kc"], a["vc"], a["dtype"], a["B"], a["C"], a["Hkv"], a["D"],
            a["bs"], a["NB"], a["maxblk"], a["stream"]]
    assert lib.paged_kv_append(*args) == status


def test_options(lib):
    assert lib.taco_attn_set_option(_lib.TACO_OPT_GRID_CTAS, 7) == _lib.TACO_OK
    assert lib.taco_attn_set_option(_lib.TACO_OPT_GRID_CTAS, 0) == _lib.TACO_OK
    assert lib.taco_attn_set_option(_lib.TACO_OPT_KERNEL, 5) == _lib.TACO_ERR_INVALID_ARG
    assert lib.taco_attn_set_option(99, 1) == _lib.TACO_ERR_INVALID_ARG
    assert lib.taco_attn_set_option(_lib.TACO_OPT_SEG_COST, 65) == _lib.TACO_ERR_INVALID_ARG
    assert lib.taco_attn_set_option(_lib.TACO_OPT_SEG_COST, -2) == _lib.TACO_ERR_INVALID_ARG
    assert lib.taco_attn_set_option(_lib.TACO_OPT_SEG_COST, 0) == _lib.TACO_OK
    assert lib.taco_attn_set_option(_lib.TACO_OPT_SEG_COST, -1) == _lib.TACO_OK
    assert lib.taco_attn_set_option(_lib.TACO_OPT_COMBINE, 3) == _lib.TACO_ERR_INVALID_ARG
    assert lib.taco_attn_set_option(_lib.TACO_OPT_COMBINE, 0) == _lib.TACO_OK


@pytest.mark.parametrize("call,status", [
    (lambda l: l.tree_mask_from_parents(None, 16, 2, 4, 16, None), _lib.TACO_ERR_INVALID_ARG),
    (lambda l: l.tree_mask_from_parents(16, 16, 2, 33, 16, None), _lib.TACO_ERR_UNSUPPORTED),
    (lambda l: l.tree_mask_from_parents(16, 16, -1, 4, 16, None), _lib.TACO_ERR_INVALID_ARG),
    (lambda l: l.logits_argmax(None, 1, 4, 100, 16, None), _lib.TACO_ERR_INVALID_ARG),
    (lambda l: l.logits_argmax(16, 5, 4, 100, 16, None), _lib.TACO_ERR_INVALID_ARG),
    (lambda l: l.logits_argmax(16, 1, 4, 0, 16, None), _lib.TACO_ERR_INVALID_ARG),
    (lambda l: l.logits_argmax(16, 1, -2, 10, 16, None), _lib.TACO_ERR_INVALID_ARG),
    (lambda l: l.tree_greedy_accept(16, 16, 16, 16, 16, 2, 0, 16, 16, 16, 16, None), _lib.TACO_ERR_UNSUPPORTED),
    (lambda l: l.tree_greedy_accept(16, 16, 16, 16, 16, 2, 40, 16, 16, 16, 16, None), _lib.TACO_ERR_UNSUPPORTED),
    (lambda l: l.tree_greedy_accept(16, None, 16, 16, 16, 2, 4, 16, 16, 16, 16, None), _lib.TACO_ERR_INVALID_ARG),
    (lambda l: l.tree_greedy_accept(16, 16, 16, 16, 16, 2, 4, 16, 16, 16, None, None), _lib.TACO_ERR_INVALID_ARG),
])
def test_acceptance_calls_reject_bad_arguments_on_host(lib, call, status):
    assert call(lib) == status
    assert lib.taco_attn_last_error().decode()


def test_acceptance_calls_with_nothing_to_do_are_no_ops(lib):
    assert lib.tree_mask_from_parents(16, 16, 0, 4, 16, None) == _lib.TACO_OK
    assert lib.logits_argmax(16, 1, 0, 100, 16, None) == _lib.TACO_OK
    assert lib.tree_greedy_accept(16, 16, 16, 16, 16, 0, 4, 16, 16, 16, 16, None) == _lib.TACO_OK


def _attn8_args(**over):
    a = dict(ks=16, vs=16)
    a.update({k: over.pop(k) for k in list(over) if k in a})
    base = _attn_args(**over)
    return base[:3] + [a["ks"], a["vs"]] + base[3:]


@pytest.mark.parametrize("over,status", [
    (dict(ks=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(vs=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(q=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(D=96), _lib.TACO_ERR_UNSUPPORTED),          # head_dim 64 or 128 only
    (dict(Hq=129 * 2, Hkv=2, C=1), _lib.TACO_ERR_UNSUPPORTED),  # G > 128: neither kernel takes it
    (dict(dtype=3), _lib.TACO_ERR_INVALID_ARG),
    (dict(k=24), _lib.TACO_ERR_INVALID_ARG),
])
def test_e4m3_attention_rejects_bad_arguments_on_host(lib, over, status):
    assert lib.paged_tree_attention_e4m3(*_attn8_args(**over)) == status
    assert lib.taco_attn_last_error().decode()


@pytest.mark.parametrize("over", [dict(D=64), dict(Hq=64, Hkv=2, C=4)])
def test_e4m3_mma_kernel_rejects_shapes_only_the_tensor_core_kernel_takes(lib, over):
    """Forcing the mma.sync kernel (head_dim 128, <= 64 packed rows for e4m3) on head_dim 64 or on
    32 x 4 packed rows is refused on the host; the automatic choice takes the tcgen05 kernel there."""
    assert lib.taco_attn_set_option(_lib.TACO_OPT_KERNEL, 1) == _lib.TACO_OK
    try:
        assert lib.paged_tree_attention_e4m3(*_attn8_args(**over)) == _lib.TACO_ERR_UNSUPPORTED
        assert "mma.sync" in lib.taco_attn_last_error().decode()
    finally:
        assert lib.taco_attn_set_option(_lib.TACO_OPT_KERNEL, 0) == _lib.TACO_OK


def test_e4m3_calls_with_empty_batch_are_no_ops(lib):
    assert lib.paged_tree_attention_e4m3(*_attn8_args(B=0)) == _lib.TACO_OK
    args = [16, 16, 16, 16, 16, 16, 16, 16, 1, 0, 4, 2, 128, 16, 40, 8, None]
    assert lib.paged_kv_append_e4m3(*args) == _lib.TACO_OK


@pytest.mark.parametrize("over,status", [
    (dict(ks=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(vs=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(kc=8), _lib.TACO_ERR_INVALID_ARG),
    (dict(D=96), _lib.TACO_ERR_UNSUPPORTED),
    (dict(dtype=2), _lib.TACO_ERR_INVALID_ARG),
])
def test_e4m3_append_rejects_bad_arguments_on_host(lib, over, status):
    a = dict(kn=16, vn=16, bt=16, so=16, ks=16, vs=16, kc=16, vc=16, dtype=1, B=2, C=4, Hkv=2, D=128, bs=16,
             NB=40, maxblk=8, stream=None)
    a.update(over)
    args = [a["kn"], a["vn"], a["bt"], a["so"], a["ks"], a["vs"], a["kc"], a["vc"], a["dtype"], a["B"], a["C"],
            a["Hkv"], a["D"], a["bs"], a["NB"], a["maxblk"], a["stream"]]
    assert lib.paged_kv_append_e4m3(*args) == status
    assert lib.taco_attn_last_error().decode()


def _prefix_args(insert, **over):
    a = dict(tok=16, st=16, bt=16, keys=16, nodes=16, cap=1024, par=16, dep=16, ntok=16, out=16, cnt=16, B=2,
             bs=16, NB=40, maxblk=8, stream=None)
    a.update(over)
    head = [a["tok"], a["st"]] + ([a["bt"]] if insert else [])
    return head + [a["keys"], a["nodes"], ctypes.c_int64(a["cap"]), a["par"], a["dep"], a["ntok"], a["out"], a["cnt"],
                   a["B"], a["bs"], a["NB"], a["maxblk"], a["stream"]]


@pytest.mark.parametrize("insert", [False, True])
@pytest.mark.parametrize("over,status", [
    (dict(tok=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(keys=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(ntok=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(keys=12), _lib.TACO_ERR_INVALID_ARG),     # not 8-byte aligned
    (dict(cap=1000), _lib.TACO_ERR_INVALID_ARG),    # not a power of two
    (dict(cap=1), _lib.TACO_ERR_INVALID_ARG),
    (dict(bs=0), _lib.TACO_ERR_UNSUPPORTED),
    (dict(bs=2048), _lib.TACO_ERR_UNSUPPORTED),
    (dict(B=-1), _lib.TACO_ERR_INVALID_ARG),
    (dict(NB=0), _lib.TACO_ERR_INVALID_ARG),
    (dict(maxblk=0), _lib.TACO_ERR_INVALID_ARG),
])
def test_prefix_calls_reject_bad_arguments_on_host(lib, insert, over, status):
    fn = lib.prefix_cache_insert if insert else lib.prefix_cache_lookup
    assert fn(*_prefix_args(insert, **over)) == status
    assert lib.taco_attn_last_error().decode()


def test_prefix_lookup_needs_out_matched_and_insert_needs_tables(lib):
    assert lib.prefix_cache_lookup(*_prefix_args(False, cnt=None)) == _lib.TACO_ERR_INVALID_ARG
    assert lib.prefix_cache_insert(*_prefix_args(True, bt=None)) == _lib.TACO_ERR_INVALID_ARG
    assert lib.prefix_cache_insert(*_prefix_args(True, cnt=None, B=0)) == _lib.TACO_OK   # out_inserted optional


def test_prefix_calls_with_empty_batch_are_no_ops(lib):
    assert lib.prefix_cache_lookup(*_prefix_args(False, B=0)) == _lib.TACO_OK
    assert lib.prefix_cache_insert(*_prefix_args(True, B=0)) == _lib.TACO_OK


@pytest.mark.parametrize("over,status", [
    (dict(h=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(cl=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(g=None), _lib.TACO_ERR_INVALID_ARG),      # global_len > 0 needs tokens
    (dict(glen=-1), _lib.TACO_ERR_INVALID_ARG),
    (dict(M=0), _lib.TACO_ERR_UNSUPPORTED),
    (dict(M=17), _lib.TACO_ERR_UNSUPPORTED),
    (dict(C=33), _lib.TACO_ERR_UNSUPPORTED),
    (dict(C=0), _lib.TACO_ERR_UNSUPPORTED),
    (dict(B=-1), _lib.TACO_ERR_INVALID_ARG),
])
def test_lookahead_propose_rejects_bad_arguments_on_host(lib, over, status):
    a = dict(h=16, st=16, g=16, glen=100, cl=16, M=4, B=2, C=16, t=16, p=16, n=16, stream=None)
    a.update(over)
    args = [a["h"], a["st"], a["g"], ctypes.c_int64(a["glen"]), a["cl"], a["M"], a["B"], a["C"], a["t"], a["p"], a["n"],
            a["stream"]]
    assert lib.lookahead_propose(*args) == status
    assert lib.taco_attn_last_error().decode()


@pytest.mark.parametrize("over,status", [
    (dict(acc=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(hit=None), _lib.TACO_ERR_INVALID_ARG),
    (dict(cmax=0), _lib.TACO_ERR_INVALID_ARG),
    (dict(alpha=1.5), _lib.TACO_ERR_INVALID_ARG),
    (dict(alpha=float("nan")), _lib.TACO_ERR_INVALID_ARG),
    (dict(bref=0), _lib.TACO_ERR_INVALID_ARG),
    (dict(B=-3), _lib.TACO_ERR_INVALID_ARG),
])
def test_copy_len_update_rejects_bad_arguments_on_host(lib, over, status):
    a = dict(acc=16, prop=16, hit=16, cl=16, B=4, cmax=8, alpha=0.5, bref=16, stream=None)
    a.update(over)
    args = [a["acc"], a["prop"], a["hit"], a["cl"], a["B"], a["cmax"], ctypes.c_float(a["alpha"]), a["bref"], a["stream"]]
    assert lib.lookahead_update_copy_len(*args) == status


def test_lookahead_calls_with_empty_batch_are_no_ops(lib):
    assert lib.lookahead_propose(16, 16, None, ctypes.c_int64(0), 16, 4, 0, 16, 16, 16, 16, None) == _lib.TACO_OK
    assert lib.lookahead_update_copy_len(16, 16, 16, 16, 0, 8, ctypes.c_float(0.5), 16, None) == _lib.TACO_OK


def test_fused_append_attention_rejects_bad_arguments_on_host(lib):
    def args(**over):
        a = dict(kn=16, vn=16)
        a.update({k: over.pop(k) for k in list(over) if k in a})
        base = _attn_args(**over)
        return [base[0], a["kn"], a["vn"]] + base[1:]
    assert lib.paged_tree_attention_append(*args(kn=None)) == _lib.TACO_ERR_INVALID_ARG
    assert lib.paged_tree_attention_append(*args(vn=None)) == _lib.TACO_ERR_INVALID_ARG
    assert lib.paged_tree_attention_append(*args(kn=24)) == _lib.TACO_ERR_INVALID_ARG   # misaligned
    assert lib.paged_tree_attention_append(*args(D=96)) == _lib.TACO_ERR_UNSUPPORTED
    assert lib.paged_tree_attention_append(*args(B=0)) == _lib.TACO_OK
