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


def pins_fail(test_module, mod, names):
    """Run every test function of test_module with the given names re-bound to mod's; True if any fails."""
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
                except Exception:
                    return True
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
    assert pins_fail(t, mutant("prefix_cache", old, new),
                     ["PrefixTree", "batch_insert_choices", "insert_batch", "lookup_batch"])


@pytest.mark.parametrize("old,new", LOOKAHEAD_MUTATIONS)
def test_lookahead_pins_catch(old, new):
    import tests.test_oracle_lookahead as t
    assert pins_fail(t, mutant("lookahead_cache", old, new),
                     ["build_forest", "longest_match", "propose", "propose_batch", "update_copy_len"])


@pytest.mark.parametrize("old,new", ACCEPT_MUTATIONS)
def test_acceptance_pins_catch(old, new):
    import tests.test_oracle_accept as t
    saved = t.ta                       # the pin module calls the oracle through this module alias
    t.ta = mutant("tree_accept", old, new)
    try:
        assert pins_fail(t, t.ta, [])
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
