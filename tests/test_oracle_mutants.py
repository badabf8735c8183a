"""The oracle's pins catch planted mistakes (no GPU).

Each case copies the oracle's C source, plants one plausible mistake in the
copy (a transposed operand, a dropped term, a wrong sign, a wrong comparison
or tie order, a dropped scale, an off-by-one window, a wrong head mapping),
builds it with gcc in a temporary folder and points the oracle module at it
for the duration of the case; at least one pin of test_oracle_pins must then
fail.  The real oracle build is never touched.
"""
import os
import shutil
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "rtp_oracle.c")

# (what the mistake is, text in the oracle, replacement, occurrences replaced)
MUTANTS = [
    ("projection: W read transposed", "Wd[d * ORC_R + c]", "Wd[c * ORC_D + d]", 1),
    ("bf16: truncation instead of nearest", "double r = rint(ldexp(a, -q));",
     "double r = trunc(ldexp(a, -q));", 1),
    ("bf16: ties away from zero", "double r = rint(ldexp(a, -q));",
     "double r = round(ldexp(a, -q));", 1),
    ("scores: first term dropped",
     "for (int c = 0; c < ORC_R; ++c)\n            acc += q[c] * orc_bf16_to_double(kr[c]);",
     "for (int c = 1; c < ORC_R; ++c)\n            acc += q[c] * orc_bf16_to_double(kr[c]);", 1),
    ("softmax: exponent sign flipped in Z", "Z += exp(s[j] - m);", "Z += exp(m - s[j]);", 1),
    ("top-p: must exceed p instead of reach it", "if (acc >= target)", "if (acc > target)", 1),
    ("top-p: ties go to the higher index", "return (x->j < y->j) ? -1 : (x->j > y->j);",
     "return (x->j > y->j) ? -1 : (x->j < y->j);", 1),
    ("top-p: kept mass not divided by Z", "*mass_frac = acc / Z;", "*mass_frac = acc;", 1),
    ("attention: logit scale dropped", "logit[a] = acc * scale;", "logit[a] = acc;", 1),
    ("attention: lse without the max", "*lse = mx + log(den);", "*lse = log(den);", 1),
    ("local: window one key too wide", "j > P - window", "j >= P - window", 1),
    ("local: sinks dropped", "if (j < n_sink || j > P - window)", "if (j > P - window)", 1),
    ("GQA: kv head by modulo", "h = row_h[r], g = h / G;", "h = row_h[r], g = h % S.Hkv;", 2),
    ("top-k: one key too many", "const int64_t kept = k < n ? k : n;",
     "const int64_t kept = k < n ? k + 1 : n;", 1),
    ("block top-p: bins walked from the bottom", "for (int64_t k = nbins - 1; k >= 0; --k) {",
     "for (int64_t k = 0; k < nbins; ++k) {", 1),
    ("block top-p: block mass from its max, not its log-sum-exp",
     "const double w = exp(lb[b] - hi);", "const double w = exp(mb[b] - hi);", 1),
    ("block top-p: threshold bin left out", "const int on = bin[b] >= kstar;",
     "const int on = bin[b] > kstar;", 1),
    ("block top-p: range from 0, not from the lowest block max",
     "floor(((mb[b] - lo) / (hi - lo)) * (double)nbins)", "floor((mb[b] / hi) * (double)nbins)",
     1),
]


def _pin_calls():
    """Every pin of test_oracle_pins as (name, zero-argument callable)."""
    calls = []
    for name in sorted(n for n in dir(pins) if n.startswith("test_")):
        fn = getattr(pins, name)
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            calls.append((name, fn))
            continue
        assert len(marks) == 1, name
        argnames, values = marks[0].args[0], marks[0].args[1]
        names = [a.strip() for a in argnames.split(",")]
        for k, val in enumerate(values):
            args = tuple(val) if len(names) > 1 else (val,)
            calls.append((f"{name}[{k}]", lambda fn=fn, kw=dict(zip(names, args)): fn(**kw)))
    return calls


def _build_mutant(tmp_path, old, new, count):
    src = open(SRC).read()
    assert src.count(old) == count, (old, src.count(old))
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-o",
                           str(lib), str(path), "-lm"])
    return str(lib)


@pytest.fixture(scope="module")
def pin_calls():
    return _pin_calls()


def test_pins_pass_on_the_oracle(pin_calls):
    """The harness itself: every collected pin passes on the unmodified oracle."""
    assert len(pin_calls) > 20
    for _, call in pin_calls:
        call()


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("what,old,new,count", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(what, old, new, count, tmp_path, monkeypatch, pin_calls):
    lib = _build_mutant(tmp_path, old, new, count)
    monkeypatch.setattr(oracle, "_lib", None)
    monkeypatch.setattr(oracle, "build", lambda force=False: lib)
    failed = []
    for name, call in pin_calls:
        try:
            call()
        except AssertionError:
            failed.append(name)
            break
    assert failed, f"no pin fails with the mistake '{what}'"
