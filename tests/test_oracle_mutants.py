"""The oracle's pins catch plausible mistakes (CPU).

Each case plants one mistake in a copy of the oracle's C source -- a wrong
divisor, a dropped term, a scale taken from the wrong array, a wrong head
routing, an off-by-one at a boundary, a swapped nibble order -- compiles the
copy, and runs the pins that cover that part of the oracle against it: at
least one must fail.  Every planted mistake keeps every memory access in
bounds (no index is changed beyond a valid one), so a copy can only compute
wrong values, never crash.  A control copy with no change passes every pin,
which shows the harness itself reports nothing spurious.
"""
import importlib
import importlib.util
import inspect
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_DIR = os.path.join(ROOT, "oracle")

INT8 = ("tests.test_oracle_pins", "tests.test_oracle_extend_pins")
INT4 = ("tests.test_oracle_int4_pins",)
KIVI = ("tests.test_oracle_kivi_pins",)

# (name, text in kv8_oracle.c, replacement, pin modules); the text occurs
# once unless `nth` picks one occurrence (0-based) of several
MUTANTS = [
    ("int8 scale divides by 128", "a / 127.0f;", "a / 128.0f;", INT8, None),
    ("int8 codes truncate", "float r = nearbyintf(y); /* default mode: ties to even */",
     "float r = truncf(y); /* default mode: ties to even */", INT8, None),
    ("K scale dropped", "double ks = (double)k_scales[base];", "double ks = 1.0;", INT8, None),
    ("V scale read from the K scales", "double vs = (double)v_scales[base];",
     "double vs = (double)k_scales[base];", INT8, None),
    ("softmax not normalised", "double w = score[t] / denom;", "double w = score[t];", INT8, None),
    ("default scale 1/d instead of 1/sqrt(d)", "softmax_scale = 1.0 / sqrt((double)head_dim);",
     "softmax_scale = 1.0 / (double)head_dim;", INT8, 0),
    ("decode heads routed modulo", "softmax_scale, b, h / group, context_lens[b],",
     "softmax_scale, b, h % num_kv_heads, context_lens[b],", INT8, None),
    ("extend heads routed modulo", "softmax_scale, b, h / group, keys, orow);",
     "softmax_scale, b, h % num_kv_heads, keys, orow);", INT8, None),
    ("extend row misses its own token", "int32_t keys = context_lens[b] - n_new + i + 1;",
     "int32_t keys = context_lens[b] - n_new + i;", INT8, None),
    ("int4 scale divides by 8", "a / 7.0f;", "a / 8.0f;", INT4, None),
    ("int4 nibbles read in the wrong order", "int nib = (j & 1) ? (byte >> 4) : (byte & 15);",
     "int nib = (j & 1) ? (byte & 15) : (byte >> 4);", INT4, None),
    ("kivi range over 4 levels", "float s = (hi - lo) / 3.0f;", "float s = (hi - lo) / 4.0f;",
     KIVI, None),
    ("kivi key zero point dropped", "(double)k_zero[page * head_dim + j];", "0.0;", KIVI, None),
    ("kivi value zero point read from the scales", "(double)v_zero[page * block_size + r];",
     "(double)v_scale[page * block_size + r];", KIVI, None),
    ("kivi first tail token read from its page", "if (t < full) {", "if (t <= full) {",
     KIVI, None),
]


def _replace(src, old, new, nth):
    if nth is None:
        assert src.count(old) == 1, old
        return src.replace(old, new)
    parts = src.split(old)
    assert len(parts) > nth + 1, old
    return old.join(parts[:nth + 1]) + new + old.join(parts[nth + 1:])


def _oracle_copy(tmp_path, src):
    """A separate instance of the oracle package bound to a copy of its C
    source (compiled into tmp_path)."""
    c_path = tmp_path / "kv8_oracle.c"
    c_path.write_text(src)
    spec = importlib.util.spec_from_file_location(
        f"oracle_copy_{tmp_path.name}", os.path.join(ORACLE_DIR, "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod._SRC = str(c_path)
    mod._LIB_PATH = str(tmp_path / "libkv8_oracle_copy.so")
    mod._lib = None
    mod.build(force=True)
    return mod


def _run_pins(mod, modules):
    """Run every pin of `modules` against `mod`; return the names that fail."""
    failed = []
    for name in modules:
        pins = importlib.import_module(name)
        for fname, fn in sorted(vars(pins).items()):
            if not fname.startswith("test_") or not callable(fn):
                continue
            assert list(inspect.signature(fn).parameters) == ["oracle_mod"], fname
            try:
                fn(mod)
            except (AssertionError, ValueError):
                failed.append(f"{name}.{fname}")
    return failed


def _source():
    with open(os.path.join(ORACLE_DIR, "kv8_oracle.c")) as f:
        return f.read()


def test_unchanged_copy_passes_every_pin(tmp_path):
    mod = _oracle_copy(tmp_path, _source())
    assert _run_pins(mod, INT8 + INT4 + KIVI) == []


@pytest.mark.parametrize("name,old,new,modules,nth", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, old, new, modules, nth):
    mod = _oracle_copy(tmp_path, _replace(_source(), old, new, nth))
    failed = _run_pins(mod, modules)
    assert failed, f"no pin caught: {name}"
