"""Mutation check of the backward-pass and warm-tier oracles' pins: every planted
slip in oracle/hga_backward.py or oracle/hga_warm.py must fail at least one pin
of tests/test_backward_pins.py or tests/test_warm_pins.py.  The oracle files are
never modified: each mutant is the edited text loaded as a separate module.

Not a slip, and so not listed: letting a step's hits into the victim order.  The
hits carry the new clock, the largest stamp, so they sort after every other slot,
and a step never has more misses than non-hit slots (requests <= slots): no
hit is ever chosen, and the edit changes no value.
"""

import importlib.util
import itertools
import os
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ORACLE_DIR = os.path.join(os.path.dirname(HERE), "oracle")

# (name, exact text in the oracle file, replacement)
BACKWARD = [
    ("value gradient without the weights",
     "dv = np.outer(w, d_out)",
     "dv = np.outer(np.ones_like(w), d_out)"),
    ("score gradient without the Delta term",
     "ds = w * (dw - float(d_out @ o))",
     "ds = w * dw"),
    ("query gradient without the softmax scale",
     "dq = (kk.T @ ds) * scale",
     "dq = kk.T @ ds"),
    ("key gradient from the output gradient",
     "dk = np.outer(ds, q_vec) * scale",
     "dk = np.outer(ds, d_out) * scale"),
    ("weight gradient through the keys",
     "dw = vv @ d_out",
     "dw = kk @ d_out"),
    ("scale sqrt(D) instead of 1/sqrt(D)",
     "scale = 1.0 / math.sqrt(q_vec.shape[0])",
     "scale = math.sqrt(q_vec.shape[0])"),
    ("key gradients summed into the first KV head",
     "dk[h, toks] += gk",
     "dk[0, toks] += gk"),
    ("query gradient stored for the group's first head",
     "dq[hh, r] = gq",
     "dq[h * g, r] = gq"),
]

WARM = [
    ("clock not advanced",
     "clock = int(stamp.max()) + 1 if M else 1",
     "clock = int(stamp.max()) if M else 1"),
    ("hits keep their old stamp",
     "    for s in hit_slots:\n        stamp[s] = clock",
     "    for s in hit_slots:\n        pass"),
    ("most recently used evicted first",
     "victims = sorted((s for s in range(M) if s not in hit_slots), key=order)",
     "victims = sorted((s for s in range(M) if s not in hit_slots), key=order, reverse=True)"),
    ("ties evict the higher id",
     "return (0, s, 0) if tag[s] < 0 else (1, int(stamp[s]), int(tag[s]))",
     "return (0, s, 0) if tag[s] < 0 else (1, int(stamp[s]), -int(tag[s]))"),
    ("empty slots taken last",
     "return (0, s, 0) if tag[s] < 0 else (1, int(stamp[s]), int(tag[s]))",
     "return (2, s, 0) if tag[s] < 0 else (1, int(stamp[s]), int(tag[s]))"),
    ("repeated ids kept",
     "if ids and gid <= ids[-1]:",
     "if ids and gid < ids[-1]:"),
    ("oldest local chunk taken as a candidate",
     "if not (sink <= c < cur - local):",
     "if not (sink <= c <= cur - local):"),
    ("slot map holds positions",
     "        row[j] = s",
     "        row[j] = j"),
]

SUITES = {
    "backward": ("hga_backward.py", "test_backward_pins.py", "BW", BACKWARD),
    "warm": ("hga_warm.py", "test_warm_pins.py", "W", WARM),
}


def _load_pins(pins_file):
    spec = importlib.util.spec_from_file_location("pins_for_mutation_" + pins_file[:-3],
                                                  os.path.join(HERE, pins_file))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _mutant(path, src: str, name: str):
    mod_name = "oracle.mutant_" + str(abs(hash(name)))
    spec = importlib.util.spec_from_loader(mod_name, loader=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"   # its relative imports resolve to the real oracle package
    sys.modules[mod_name] = mod
    try:
        exec(compile(src, path + " [" + name + "]", "exec"), mod.__dict__)
    finally:
        sys.modules.pop(mod_name, None)
    return mod


def _cases(fn):
    axes = []
    for mark in getattr(fn, "pytestmark", []):
        if mark.name != "parametrize":
            continue
        names = [s.strip() for s in mark.args[0].split(",")]
        values = [v if len(names) > 1 else (v,) for v in mark.args[1]]
        axes.append([dict(zip(names, v)) for v in values])
    for combo in itertools.product(*axes):
        kw = {}
        for part in combo:
            kw.update(part)
        yield kw


def _pins_fail(pins, attr, mutant):
    setattr(pins, attr, mutant)
    for name, fn in vars(pins).items():
        if not (name.startswith("test_") and callable(fn)):
            continue
        for kw in _cases(fn):
            try:
                fn(**kw)
            except Exception:  # noqa: BLE001 - any failure of a pin kills the mutant
                return name
    return None


@pytest.mark.parametrize("suite", list(SUITES))
def test_mutations_apply_once_and_the_unmutated_oracle_passes(suite):
    oracle, pins_file, attr, muts = SUITES[suite]
    path = os.path.join(ORACLE_DIR, oracle)
    src = open(path).read()
    for name, old, _ in muts:
        assert src.count(old) == 1, f"mutation {name!r} does not match {oracle} once"
    assert _pins_fail(_load_pins(pins_file), attr, _mutant(path, src, "original")) is None


@pytest.mark.parametrize("suite,name,old,new",
                         [(s, *m) for s, v in SUITES.items() for m in v[3]],
                         ids=[f"{s}: {m[0]}" for s, v in SUITES.items() for m in v[3]])
def test_every_planted_slip_fails_a_pin(suite, name, old, new):
    oracle, pins_file, attr, _ = SUITES[suite]
    path = os.path.join(ORACLE_DIR, oracle)
    src = open(path).read()
    pins = _load_pins(pins_file)
    assert _pins_fail(pins, attr, _mutant(path, src.replace(old, new), name)) is not None, \
        f"no pin catches: {name}"
