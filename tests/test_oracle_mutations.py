"""Mutation check of the oracle pins: every planted slip must fail at least one pin.

Each mutation below edits the oracle's source text in one place - a plausible
mistake in restating the HGA mechanism (a wrong span centre, a rotation sign,
the pair layout, the high/low split, the candidate window, the tie rule, the
GQA mean, causality, the softmax scale, a missing mean) - loads the edited text
as a separate module, and runs every pin of test_oracle_pins.py against it in
this process.  The test passes when every mutant fails at least one pin.  The
oracle file itself is never modified.

Not a slip, and so not listed: passing span_summary another start position t0
for the same keys.  The start cancels between the un-rotation at t0 + m and the
re-rotation at the centre t0 + (L-1)/2, R(t0 + (L-1)/2) R(-(t0 + m)) =
R((L-1)/2 - m), so such an edit changes no value (the pin
test_span_summary_start_position_cancels states exactly this).  The position
slips that do change values - a wrong centre, re-rotation at the span start,
rows built from the wrong tokens - are listed.
"""

import importlib.util
import itertools
import os
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ORACLE = os.path.join(os.path.dirname(HERE), "oracle", "hga_oracle.py")

# (name, exact text in the oracle, replacement)
MUTATIONS = [
    ("group row from its chunk's first tokens",
     "group_sum[c, gi] = span_summary(k_rot[g0:g0 + prm.group], g0,",
     "group_sum[c, gi] = span_summary(k_rot[c0:c0 + prm.group], g0,"),
    ("chunk row from the tokens one group later",
     "chunk_sum[c] = span_summary(k_rot[c0:c0 + prm.chunk], c0, prm.n_high_pairs,",
     "chunk_sum[c] = span_summary(k_rot[c0 + prm.group:c0 + prm.chunk + prm.group], c0, "
     "prm.n_high_pairs,"),
    ("centre off by half a token",
     "centre = t0 + (length - 1) / 2.0",
     "centre = t0 + length / 2.0"),
    ("low pairs rotated at the span start",
     "low_part = rope_apply(mean_raw[None, :], [centre], theta)[0]",
     "low_part = rope_apply(mean_raw[None, :], [t0], theta)[0]"),
    ("un-rotation with the wrong sign",
     "raw = rope_apply(k_rot_span, -positions, theta)",
     "raw = rope_apply(k_rot_span, positions, theta)"),
    ("interleaved instead of rotate-half pairs",
     "a, b = x[..., :p], x[..., p:]",
     "a, b = x[..., 0::2], x[..., 1::2]"),
    ("rotation sense flipped",
     "return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)",
     "return np.concatenate([a * c + b * s, b * c - a * s], axis=-1)"),
    ("frequencies theta^(-i/D)",
     "-2.0 * np.arange(pairs, dtype=np.float64) / head_dim",
     "-1.0 * np.arange(pairs, dtype=np.float64) / head_dim"),
    ("high-frequency pairs taken from the end",
     "pair_is_high = np.arange(p) < n_high_pairs",
     "pair_is_high = np.arange(p) >= p - n_high_pairs"),
    ("low-pair sum without the mean",
     "mean_raw = raw.mean(axis=0)",
     "mean_raw = raw.sum(axis=0)"),
    ("high-pair mean over L-1",
     "mean_rotated = k_rot_span.mean(axis=0)",
     "mean_rotated = k_rot_span.sum(axis=0) / (length - 1)"),
    ("incomplete chunk rows computed",
     "if c0 + prm.chunk <= n_valid:",
     "if c0 < n_valid:"),
    ("routing query from the first head only",
     "return q_rows.reshape(-1, q_rows.shape[-1]).mean(axis=0)",
     "return q_rows.reshape(-1, q_rows.shape[-1])[0]"),
    ("candidate window includes the oldest local chunk",
     "return list(range(prm.sink, max(prm.sink, cur - prm.local)))",
     "return list(range(prm.sink, max(prm.sink, cur - prm.local + 1)))"),
    ("sink chunks start at 1",
     "sink = set(range(0, min(prm.sink, cur + 1)))",
     "sink = set(range(1, min(prm.sink, cur + 1)))"),
    ("local window one chunk short",
     "recent = set(range(max(0, cur - prm.local), cur + 1))",
     "recent = set(range(max(0, cur - prm.local + 1), cur + 1))"),
    ("ties to the higher index",
     "key=lambda i: (-scores[i], ids[i])",
     "key=lambda i: (-scores[i], -ids[i])"),
    ("selection returned in score order",
     "chosen = sorted(ids[i] for i in order[:k])",
     "chosen = [ids[i] for i in order[:k]]"),
    ("wrong global group id",
     "cand.append(c * ng + gi)",
     "cand.append(gi * ng + c)"),
    ("query sees one token past itself",
     "if t <= query_pos), dtype=np.int64)",
     "if t <= query_pos + 1), dtype=np.int64)"),
    ("softmax scale 1/D",
     "s = kk @ q_vec / math.sqrt(q_vec.shape[0])",
     "s = kk @ q_vec / q_vec.shape[0]"),
    ("LSE without the log",
     "return w @ vv, m + math.log(z), w",
     "return w @ vv, m + z, w"),
    ("current chunk taken as pos // group",
     "return [(0, 1, pos_last // chunk)]",
     "return [(0, 1, pos_last // (chunk // 2))]"),
]


def _load_pins():
    spec = importlib.util.spec_from_file_location("hga_oracle_pins_for_mutation",
                                                  os.path.join(HERE, "test_oracle_pins.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _mutant(src: str, name: str):
    mod_name = "hga_oracle_mutant_" + str(abs(hash(name)))
    spec = importlib.util.spec_from_loader(mod_name, loader=None)
    mod = importlib.util.module_from_spec(spec)
    sys.modules[mod_name] = mod  # dataclasses look their module up here
    try:
        exec(compile(src, ORACLE + " [" + name + "]", "exec"), mod.__dict__)
    finally:
        sys.modules.pop(mod_name, None)
    return mod


def _cases(fn):
    """Every parameter combination of a pin (its pytest.mark.parametrize marks)."""
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


def _pins_fail(pins, mutant) -> str | None:
    """Name of the first pin the mutant fails, or None when it passes them all."""
    pins.O = mutant
    for name, fn in vars(pins).items():
        if not (name.startswith("test_") and callable(fn)):
            continue
        for kw in _cases(fn):
            try:
                fn(**kw)
            except Exception:  # noqa: BLE001 - any failure of a pin kills the mutant
                return f"{name}{kw if kw else ''}"
    return None


def test_mutations_apply_to_the_oracle_text_once():
    src = open(ORACLE).read()
    for name, old, _ in MUTATIONS:
        assert src.count(old) == 1, f"mutation {name!r} does not match the oracle text once"


def test_unmutated_oracle_passes_every_pin():
    pins = _load_pins()
    assert _pins_fail(pins, _mutant(open(ORACLE).read(), "original")) is None


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_every_planted_slip_fails_a_pin(name, old, new):
    src = open(ORACLE).read()
    assert src.count(old) == 1
    pins = _load_pins()
    assert _pins_fail(pins, _mutant(src.replace(old, new), name)) is not None, \
        f"no pin catches: {name}"
