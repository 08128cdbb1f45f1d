"""Each plausible mistake planted in the oracle (a flipped sign, a dropped
term, a wrong index or axis, a transposed operand) makes at least one of
its pins fail.  The mistake is planted in a copy of the oracle's source,
executed as a separate module, and the pins of tests/test_oracle_pins.py
are run against that copy (on the CPU; the oracle itself is not changed)."""
import os
import types

import pytest

from tests import test_oracle_pins as pins

ORACLE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "mova_oracle.py")

# (name, text in the oracle, replacement): each text occurs exactly once.
MUTATIONS = [
    ("sigmoid sign", "return 1.0 / (1.0 + np.exp(-z))", "return 1.0 / (1.0 + np.exp(z))"),
    ("SiLU sign", "return h * sigmoid(h)", "return h * sigmoid(-h)"),
    ("SiLU missing", "v[rows] += w[rows, slot][:, None] * silu(h)", "v[rows] += w[rows, slot][:, None] * h"),
    ("top-k ascending", 'order = np.argsort(-b, axis=1, kind="stable")', 'order = np.argsort(b, axis=1, kind="stable")'),
    ("top-k off by one", "return order[:, :k]", "return order[:, 1:k + 1]"),
    ("top-k slots reversed", "return order[:, :k]", "return order[:, :k][:, ::-1]"),
    ("ties to the higher index", 'order = np.argsort(-b, axis=1, kind="stable")',
     'order = (b.shape[1] - 1) - np.argsort(-b[:, ::-1], axis=1, kind="stable")'),
    ("bias on the logits", "b = s + br[None, :]", "b = sigmoid(logits + br[None, :])"),
    ("bias doubled", "b = s + br[None, :]", "b = s + 2 * br[None, :]"),
    ("weights from biased scores", "s_sel = np.take_along_axis(s, idx, axis=1)\n    w = scale",
     "s_sel = np.take_along_axis(b, idx, axis=1)\n    w = scale"),
    ("no renormalisation", "w = scale * s_sel / s_sel.sum(axis=1, keepdims=True)", "w = scale * s_sel"),
    ("renormalised over tokens", "w = scale * s_sel / s_sel.sum(axis=1, keepdims=True)",
     "w = scale * s_sel / s_sel.sum(axis=0, keepdims=True)"),
    ("no scale in route", "w = scale * s_sel / s_sel.sum(axis=1, keepdims=True)",
     "w = s_sel / s_sel.sum(axis=1, keepdims=True)"),
    ("no scale in weights_for", "return scale * s_sel / s_sel.sum(axis=1, keepdims=True)",
     "return s_sel / s_sel.sum(axis=1, keepdims=True)"),
    ("slot weights swapped", "v[rows] += w[rows, slot][:, None] * silu(h)",
     "v[rows] += w[rows, (slot + 1) % k][:, None] * silu(h)"),
    ("every slot uses slot 0's experts",
     "for e in np.unique(idx[:, slot]):\n            rows = np.nonzero(idx[:, slot] == e)[0]",
     "for e in np.unique(idx[:, 0]):\n            rows = np.nonzero(idx[:, 0] == e)[0]"),
    ("router operand reversed along d", "return x @ Wr.T", "return x[:, ::-1] @ Wr.T"),
    ("bf16 bits shifted", "<< np.uint32(16)", "<< np.uint32(15)"),
    ("fp16 read as bf16 bits", 'if dtype == "bf16":', 'if dtype in ("bf16", "f16"):'),
    ("grouping in descending expert order", 'perm = np.argsort(flat, kind="stable")',
     'perm = np.argsort(-flat, kind="stable")'),
    ("pos not the inverse of perm", "pos[perm] = np.arange(perm.size, dtype=np.int64)", "pos = perm.copy()"),
    ("inclusive offsets", "offsets[1:] = np.cumsum(counts)", "offsets[:-1] = np.cumsum(counts)"),
    ("MAC count without k", "return k * d * n", "return d * n"),
    ("heads reshaped transposed", "return v.reshape(T, n // head_dim, head_dim)",
     "return v.reshape(T, head_dim, n // head_dim).transpose(0, 2, 1)"),
    ("partitions not rounded to fp32",
     ".astype(np.float32)\n        acc = part if acc is None else (acc + part).astype(np.float32)",
     ".astype(np.float64)\n        acc = part if acc is None else (acc + part)"),
    ("partitions strided instead of halves",
     "part = (x[:, p * step:(p + 1) * step] @ Wr[:, p * step:(p + 1) * step].T)",
     "part = (x[:, p::partitions] @ Wr[:, p::partitions].T)"),
    ("attend: query head onto the wrong KV head", "o[h] = probs[h].astype(np.float64) @ V[:, h // G, :]",
     "o[h] = probs[h].astype(np.float64) @ V[:, h % V.shape[1], :]"),
    ("attend: another head's probabilities", "o[h] = probs[h].astype(np.float64) @ V[:, h // G, :]",
     "o[h] = probs[H - 1 - h].astype(np.float64) @ V[:, h // G, :]"),
    ("attend: routing weights dropped", "V = as_gqa(combine(x, idx, w, Wv, wv_dtype), head_dim)",
     "V = as_gqa(combine(x, idx, np.ones_like(w), Wv, wv_dtype), head_dim)"),
]


def _pin_calls():
    """Every pin test with every parameter combination, as (name, kwargs)."""
    calls = []
    for name in sorted(dir(pins)):
        if not name.startswith("test_"):
            continue
        fn = getattr(pins, name)
        combos = [{}]
        for mark in getattr(fn, "pytestmark", []):
            if mark.name != "parametrize":
                continue
            argnames = [a.strip() for a in mark.args[0].split(",")]
            new = []
            for c in combos:
                for val in mark.args[1]:
                    vals = tuple(val) if len(argnames) > 1 else (val,)
                    new.append({**c, **dict(zip(argnames, vals))})
            combos = new
        calls.extend((name, c) for c in combos)
    return calls


def _first_failing_pin(module):
    saved = pins.O
    pins.O = module
    try:
        for name, kwargs in _pin_calls():
            try:
                getattr(pins, name)(**kwargs)
            except Exception:  # an assertion or a crash: the pin catches the mistake
                return name
        return None
    finally:
        pins.O = saved


def _mutant(old, new):
    with open(ORACLE) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation anchor must occur once: {old!r}"
    mod = types.ModuleType("mova_oracle_mutant")
    exec(compile(src.replace(old, new), "mova_oracle_mutant.py", "exec"), mod.__dict__)
    return mod


def test_unmutated_oracle_passes_every_pin():
    with open(ORACLE) as f:
        src = f.read()
    mod = types.ModuleType("mova_oracle_copy")
    exec(compile(src, "mova_oracle_copy.py", "exec"), mod.__dict__)
    assert _first_failing_pin(mod) is None


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutation_is_caught(name, old, new):
    assert _first_failing_pin(_mutant(old, new)) is not None, f"no pin catches: {name}"
