"""The oracle's pins catch plausible mistakes in the oracle.

Each case below plants one mistake in a copy of ``oracle/sdl_oracle.c``: a
dropped term, a wrong index or head mapping, a transposed operand, a changed
rounding or tie rule.  The copy is built with gcc into a temporary directory
and loaded in place of the oracle.  Then every pin of
``tests/test_oracle_pins.py`` and ``tests/test_oracle_col_pins.py`` runs
against it.  The pins come from freshly loaded copies of those modules, so
their random inputs match a normal run.  At least one pin must fail for every
mistake: a pin set that passed a wrong oracle would prove nothing about the
right one.  Every mistake planted here keeps the oracle's reads and writes
inside its buffers, so a mistake is caught by a pin and not by a crash.
"""
import importlib.util
import inspect
import os

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
PIN_FILES = ("test_oracle_pins.py", "test_oracle_col_pins.py")

# (name, text in the oracle, replacement, occurrences of the text)
MUTANTS = [
    # block means
    ("pool divides by bs + 1", "= s / (double)bs;", "= s / (double)(bs + 1);", 1),
    ("pool drops a block's last token", "t < (i + 1) * bs; ++t) s +=",
     "t < (i + 1) * bs - 1; ++t) s +=", 1),
    # block scores
    ("scores drop the scale", "z[j] = scale * s;", "z[j] = s;", 1),
    ("scores map query heads to KV heads by modulo",
     "int kh = h / g;\n      for (int i = 0; i < nb; ++i) {\n        const double* qi = qb",
     "int kh = h % Hkv;\n      for (int i = 0; i < nb; ++i) {\n        const double* qi = qb", 1),
    ("scores stored transposed", "for (int j = 0; j < nb; ++j) row[j] = z[j] / sum;",
     "for (int j = 0; j < nb; ++j) P[(((int64_t)b * H + h) * nb + j) * nb + i] = z[j] / sum;", 1),
    ("scores softmax unnormalised", "row[j] = z[j] / sum;", "row[j] = z[j];", 1),
    # budget and selection
    ("budget truncates instead of rounding", "floor((1.0 - sparsity) * total + 0.5)",
     "floor((1.0 - sparsity) * total)", 1),
    ("one block too few kept", "int64_t k = kb - (int64_t)H * nb;",
     "int64_t k = kb - (int64_t)H * nb - 1;", 1),
    ("ties go to the higher flat index", "return (x->idx > y->idx) - (x->idx < y->idx);",
     "return (x->idx < y->idx) - (x->idx > y->idx);", 1),
    ("smallest scores kept", "if (x->p > y->p) return -1;\n  if (x->p < y->p) return 1;",
     "if (x->p < y->p) return -1;\n  if (x->p > y->p) return 1;", 1),
    ("anti-diagonal forced instead of the diagonal",
     "if (i == j) {\n            mask[flat] = 1;",
     "if (i == nb - 1 - j) {\n            mask[flat] = 1;", 1),
    # block-sparse attention
    ("attention drops the scale", "x[u] = j->scale * s;", "x[u] = s;", 1),
    ("attention reads the mask transposed", "* nb + i) * nb + jb]", "* nb + jb) * nb + i]", 2),
    ("attention not normalised", "j->O[r * d + c] = n ? acc[c] / l : 0.0;",
     "j->O[r * d + c] = n ? acc[c] : 0.0;", 1),
    ("attention maps query heads to KV heads by modulo", "int kh = h / g, i = t / j->bs;",
     "int kh = h % j->Hkv, i = t / j->bs;", 1),
    ("attention LSE drops the maximum", "j->lse[r] = n ? m + log(l) : -INFINITY;",
     "j->lse[r] = n ? log(l) : -INFINITY;", 1),
    ("attention skips a kept block's last key",
     "for (int u = jb * j->bs; u < (jb + 1) * j->bs; ++u) {\n        double p",
     "for (int u = jb * j->bs; u < (jb + 1) * j->bs - 1; ++u) {\n        double p", 1),
    # column-sparse path
    ("column budget truncates", "floor((1.0 - sparsity) * (double)L / 64.0 + 0.5)",
     "floor((1.0 - sparsity) * (double)L / 64.0)", 1),
    ("column scores not averaged over query blocks", "row[u] += z[u] / sum / (double)nb;",
     "row[u] += z[u] / sum;", 1),
    ("column scores drop the scale", "z[u] = scale * s;", "z[u] = s;", 1),
    ("column ties go to the higher column", "return (x->u > y->u) - (x->u < y->u);",
     "return (x->u < y->u) - (x->u > y->u);", 1),
    ("columns not listed in ascending order",
     "qsort(pick, (size_t)Lc, sizeof(int), int_cmp);", ";", 1),
    ("column attention drops the scale", "x[x_] = j->scale * s;", "x[x_] = s;", 1),
    ("column attention maps heads by modulo",
     "int kh = h / g;\n    const int32_t* cl", "int kh = h % j->Hkv;\n    const int32_t* cl", 1),
    ("column attention not normalised", "j->O[r * d + c] = acc[c] / l;",
     "j->O[r * d + c] = acc[c];", 1),
]


def _fresh_pins():
    """Every pin as (name, callable taking no arguments), from new module copies."""
    out = []
    for i, fname in enumerate(PIN_FILES):
        spec = importlib.util.spec_from_file_location(f"_pins_copy_{i}",
                                                      os.path.join(HERE, fname))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        for name, fn in inspect.getmembers(mod, inspect.isfunction):
            if not name.startswith("test_") or fn.__module__ != mod.__name__:
                continue
            marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
            if not marks:
                assert not inspect.signature(fn).parameters, name
                out.append((name, fn))
                continue
            assert len(marks) == 1, name
            argnames = [a.strip() for a in marks[0].args[0].split(",")]
            for values in marks[0].args[1]:
                values = values if isinstance(values, (tuple, list)) else (values,)
                out.append((f"{name}{list(values)}",
                            lambda fn=fn, kw=dict(zip(argnames, values)): fn(**kw)))
    return out


def _failing_pins():
    failed = []
    for name, call in _fresh_pins():
        try:
            call()
        except (AssertionError, ValueError, RuntimeError):
            failed.append(name)
    return failed


def _use_source(monkeypatch, tmp_path, text):
    src = tmp_path / "sdl_oracle.c"
    src.write_text(text)
    monkeypatch.setattr(oracle, "_SRC", str(src))
    monkeypatch.setattr(oracle, "_SO", str(tmp_path / "libsdl_oracle.so"))
    monkeypatch.setattr(oracle, "_lib", None)
    oracle.lib()  # builds the copy; a mistake that does not compile fails here


def test_unchanged_copy_passes_every_pin(monkeypatch, tmp_path):
    with open(oracle._SRC) as f:
        _use_source(monkeypatch, tmp_path, f.read())
    assert _failing_pins() == []


@pytest.mark.parametrize("name,old,new,count", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(monkeypatch, tmp_path, name, old, new, count):
    with open(oracle._SRC) as f:
        text = f.read()
    assert text.count(old) == count, f"{name}: the text to change was not found as expected"
    _use_source(monkeypatch, tmp_path, text.replace(old, new))
    assert _failing_pins(), f"no pin fails when the oracle has: {name}"
