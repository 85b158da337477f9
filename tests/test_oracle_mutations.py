"""Mutation check of the pins (CPU only): each case plants one plausible mistake in a private copy of an
oracle module (a source edit; the real module is untouched), points the pin tests at the copy, and
requires at least one pin to fail."""
import importlib.util
import inspect
import os
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def mutant(module_name: str, old: str, new: str) -> types.ModuleType:
    path = os.path.join(ROOT, "oracle", module_name + ".py")
    src = open(path).read()
    assert src.count(old) >= 1, f"mutation site not found: {old!r}"
    mod = types.ModuleType(f"oracle._mutant_{module_name}")
    mod.__file__ = path
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new, 1), path, "exec"), mod.__dict__)
    return mod


def pins_fail(test_module, mod, names, mutated_file=None):
    """Run every test function of test_module with the given names re-bound to mod's; True if any fails.

    A pin fails by an assertion. Any other exception counts as a failure only when it was raised while
    running the mutated oracle source (a frame of mutated_file on its traceback, e.g. an index the
    mutation pushed out of range); anywhere else it is a fault of the harness or of the pin itself and
    propagates, so that a broken harness cannot pass for a caught mutant."""
    saved = {n: getattr(test_module, n) for n in names}
    try:
        for n in names:
            setattr(test_module, n, getattr(mod, n))
        for fname, fn in inspect.getmembers(test_module, inspect.isfunction):
            if not fname.startswith("test_"):
                continue
            params = inspect.signature(fn).parameters
            marks = getattr(fn, "pytestmark", [])
            cases = [()]
            for m in marks:
                if m.name == "parametrize":
                    argnames = [a.strip() for a in m.args[0].split(",")] if isinstance(m.args[0], str) else list(m.args[0])
                    new_cases = []
                    for c in cases:
                        for v in m.args[1]:
                            v = v if isinstance(v, tuple) and len(argnames) > 1 else (v,)
                            new_cases.append(c + tuple(zip(argnames, v)))
                    cases = new_cases
            for c in cases:
                kwargs = dict(c)
                if set(kwargs) != set(params):
                    continue
                try:
                    fn(**kwargs)
                except AssertionError:
                    return True
                except Exception as e:
                    tb, files = e.__traceback__, set()
                    while tb is not None:
                        files.add(tb.tb_frame.f_code.co_filename)
                        tb = tb.tb_next
                    if mutated_file is not None and mutated_file in files:
                        return True
                    raise
        return False
    finally:
        for n, v in saved.items():
            setattr(test_module, n, v)


PREFIX_MUTATIONS = [
    ("for j in range(len(toks) // self.bs)]", "for j in range((len(toks) + self.bs - 1) // self.bs)]"),  # partial blocks
    ('node = {"block": int(blocks[j]), "children": {}}', 'node = {"block": int(blocks[j]), "children": {}}; level = {}'),
    ('out.append(node["block"])', "out.append(int(blocks[j]))"),                                           # own block
    ('level = node["children"]\n        return path', 'level = self.children\n        return path'),      # flat levels
]

LOOKAHEAD_MUTATIONS = [
    ("best_m, best = m, sorted(ends, reverse=True)", "best_m, best = m, sorted(ends)"),                     # oldest first
    ("        if int(t) < 0:", "        if int(t) < -1:"),                                                  # separators copied
    ("    paths += [continuation(global_cache, e, copy_len) for e in ends_g]",
     "    paths = [continuation(global_cache, e, copy_len) for e in ends_g] + paths"),                       # global first
    ("                if len(tokens) >= C:", "                if len(tokens) > C:"),                         # budget + 1
    ("    x = f(copy_max) * new_hit * scale + f(0.5)", "    x = f(copy_max) * new_hit * scale"),             # no rounding
    ("        if ends:", "        if ends and m == 1:"),                                                      # shortest match
]

ACCEPT_MUTATIONS = [
    ("row = 0 if p < 0 else p + 1", "row = 0 if p < 0 else p"),                                               # wrong logits row
    ("and len(chain) > best_depth", "and len(chain) >= best_depth"),                                          # ties to the last
    ("slots[b, j] = P + d", "slots[b, j] = P + d + 1"),                                                       # off-by-one slot
    ("bonus[b] = int(target_argmax[b, 0 if best < 0 else best + 1])", "bonus[b] = int(target_argmax[b, 0])"),
]


@pytest.mark.parametrize("old,new", PREFIX_MUTATIONS)
def test_prefix_pins_catch(old, new):
    import tests.test_oracle_prefix as t
    m = mutant("prefix_cache", old, new)
    assert pins_fail(t, m, ["PrefixTree", "batch_insert_choices", "insert_batch", "lookup_batch"], m.__file__)


@pytest.mark.parametrize("old,new", LOOKAHEAD_MUTATIONS)
def test_lookahead_pins_catch(old, new):
    import tests.test_oracle_lookahead as t
    m = mutant("lookahead_cache", old, new)
    assert pins_fail(t, m, ["build_forest", "longest_match", "propose", "propose_batch", "update_copy_len"],
                     m.__file__)


@pytest.mark.parametrize("old,new", ACCEPT_MUTATIONS)
def test_acceptance_pins_catch(old, new):
    import tests.test_oracle_accept as t
    saved = t.ta                       # the pin module calls the oracle through this module alias
    t.ta = mutant("tree_accept", old, new)
    try:
        assert pins_fail(t, t.ta, [], t.ta.__file__)
    finally:
        t.ta = saved


def test_unmutated_oracles_pass_their_pins():
    import tests.test_oracle_accept as ta_pins
    import tests.test_oracle_lookahead as tl
    import tests.test_oracle_prefix as tp
    from oracle import lookahead_cache, prefix_cache
    assert not pins_fail(tp, prefix_cache, ["PrefixTree", "batch_insert_choices", "insert_batch", "lookup_batch"])
    assert not pins_fail(tl, lookahead_cache,
                         ["build_forest", "longest_match", "propose", "propose_batch", "update_copy_len"])
    assert not pins_fail(ta_pins, ta_pins.ta, [])


ATTENTION_MUTATIONS = [
    ("for h in range(g * G, (g + 1) * G)]", "for h in range(g, Hq, Hkv)]"),                       # wrong GQA map
    ("s = scale * (keys @ q_row)", "s = (keys @ q_row)"),                                         # dropped scale
    ("if (int(mask_word) >> j) & 1:", "if (int(mask_word) >> (n_cand - 1 - j)) & 1:"),            # reversed bits
    ("vis = list(range(P))", "vis = list(range(P + 1))"),                                         # off-by-one prefix
    ("kc[phys, h, s % bs, :] = k_new[b, i, h, :]", "kc[phys, h, (s + 1) % bs, :] = k_new[b, i, h, :]"),  # slot
    ("vc[phys, h, s % bs, :] = v_new[b, i, h, :]", "vc[phys, h, s % bs, :] = v_new[b, i, 0, :]"),  # append head
    ("return np.zeros(values.shape[-1], dtype=np.float64)", "return np.ones(values.shape[-1], dtype=np.float64)"),
    ("phys = int(table_row[p // block_size])", "phys = int(table_row[p // block_size]) if p else 0"),  # table walk
]

FP8_MUTATIONS = [
    ("c = lo if (lo & 1) == 0 else hi", "c = lo"),                                                 # ties down
    ("a = min(abs(v), E4M3_MAX)", "a = abs(v)"),                                                   # no saturation
    ("if np.signbit(v):", "if v < 0:"),                                                            # -0 loses its sign
    ("sub = sign * (m / 8.0) * 2.0 ** -6", "sub = sign * (m / 8.0) * 2.0 ** -7"),                 # subnormal scale
    ("flat_o[k] = 0x7F", "flat_o[k] = 0xFF"),                                                      # NaN code
]

_ATTN_NAMES = ("gather_sequence_kv", "paged_kv_append", "paged_tree_attention", "softmax_attend", "visible_positions",
               "widen_to_f64", "within_tolerance")


def _oracle_with(mod):
    import oracle
    ns = types.SimpleNamespace(**{k: getattr(oracle, k) for k in dir(oracle) if not k.startswith("__")})
    for n in _ATTN_NAMES:
        setattr(ns, n, getattr(mod, n))
    return ns


@pytest.mark.parametrize("old,new", ATTENTION_MUTATIONS)
def test_attention_pins_catch(old, new):
    import tests.test_oracle as t
    saved = t.oracle
    m = mutant("paged_attention", old, new)
    t.oracle = _oracle_with(m)
    try:
        assert pins_fail(t, None, [], m.__file__)
    finally:
        t.oracle = saved


@pytest.mark.parametrize("old,new", FP8_MUTATIONS)
def test_fp8_pins_catch(old, new):
    import tests.test_oracle_fp8 as t
    saved = t.fp8
    t.fp8 = mutant("fp8", old, new)
    try:
        assert pins_fail(t, None, [], t.fp8.__file__)
    finally:
        t.fp8 = saved


def test_unmutated_attention_and_fp8_oracles_pass_their_pins():
    import tests.test_oracle as t_attn
    import tests.test_oracle_fp8 as t_fp8
    assert not pins_fail(t_attn, None, [])
    assert not pins_fail(t_fp8, None, [])
