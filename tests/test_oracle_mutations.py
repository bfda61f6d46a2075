"""Plant plausible mistakes in copies of the CPU oracle and check that each one
fails at least one pin (so the pins do constrain every step of the oracle).

The mistakes are planted in the C source of a temporary copy, on the CPU; the
real oracle is never modified.  Each pin runs on a mutant in a child process,
since a broken copy may also crash; a mutant counts as caught only when a pin's
assertion fails (a crash moves on to the next pin).
"""
import os
import subprocess
import sys
import tempfile

import pytest

import oracle

_WRITE = "    /* gated delta write on the W selected slots (item 3) */\n"
_READ = "    /* sparse read after the write (item 4) */\n"
_READ_END = "    if (io->o)\n"


def _swap_read_write(src):
    i, j, k = src.index(_WRITE), src.index(_READ), src.index(_READ_END)
    return src[:i] + src[j:k] + src[i:j] + src[k:]


MUTANTS = {
    "second-half-uses-first-half": lambda s: s.replace(
        "b += (double)x[dh + c] * (double)C2[", "b += (double)x[c] * (double)C2["),
    "halves-meet-swapped-codebooks": lambda s: s.replace(
        "a += (double)x[c] * (double)C1[", "a += (double)x[c] * (double)C2[").replace(
        "b += (double)x[dh + c] * (double)C2[", "b += (double)x[dh + c] * (double)C1["),
    "slot-numbering-transposed": lambda s: s.replace(
        "c->slot = (int64_t)w->h1[a].id * n + w->h2[b].id;",
        "c->slot = (int64_t)w->h2[b].id * n + w->h1[a].id;"),
    "slot-tie-break-reversed": lambda s: s.replace(
        "return (a->slot < b->slot) ? -1 : (a->slot > b->slot);",
        "return (a->slot > b->slot) ? -1 : (a->slot < b->slot);"),
    "half-tie-break-reversed": lambda s: s.replace(
        "return (a->id < b->id) ? -1 : (a->id > b->id);",
        "return (a->id > b->id) ? -1 : (a->id < b->id);"),
    "half-topk-keeps-smallest": lambda s: s.replace(
        "  if (a->s > b->s) return -1;\n  if (a->s < b->s) return 1;\n  return (a->id",
        "  if (a->s < b->s) return -1;\n  if (a->s > b->s) return 1;\n  return (a->id", 1),
    "candidate-grid-short-by-one": lambda s: s.replace(
        "for (int b = 0; b < k; ++b) {", "for (int b = 0; b + 1 < k; ++b) {"),
    "forget-gate-dropped": lambda s: s.replace(
        "const double mt = a * (double)row[col];", "const double mt = (double)row[col];"),
    "forget-gate-on-new-value": lambda s: s.replace(
        "row[col] = (float)((1.0 - c) * mt + c * (double)vt[col]);",
        "row[col] = (float)(a * ((1.0 - c) * (double)row[col] + c * (double)vt[col]));"),
    "delta-sign-flipped": lambda s: s.replace(
        "row[col] = (float)((1.0 - c) * mt + c * (double)vt[col]);",
        "row[col] = (float)((1.0 + c) * mt - c * (double)vt[col]);"),
    "beta-dropped": lambda s: s.replace(
        "const double c = be * ww[j];", "const double c = ww[j];"),
    "uniform-weights": lambda s: s.replace(
        "wt_out[j] = exp((double)w->cand[j].s - m) / z;", "wt_out[j] = 1.0 / n_sel;"),
    "softmax-of-negated-scores": lambda s: s.replace(
        "wt_out[j] = exp((double)w->cand[j].s - m) / z;",
        "wt_out[j] = exp(m - (double)w->cand[j].s) / z;"),
    "read-before-write": _swap_read_write,
    "read-uses-write-weights": lambda s: s.replace(
        "acc[col] += rw[j] * (double)row[col];", "acc[col] += ww[j % d->W] * (double)row[col];"),
    "near-tie-threshold-1e-3": lambda s: s.replace(
        "return fabs(a - b) < 1e-5 * m;", "return fabs(a - b) < 1e-3 * m;"),
    "near-tie-never-flagged": lambda s: s.replace(
        "return fabs(a - b) < 1e-5 * m;", "return 0 * m * a * b;"),
    "near-tie-on-float32-scores": lambda s: s.replace(
        "near_tie(w->cand[n_sel - 1].s64, w->cand[n_sel].s64)",
        "near_tie(w->cand[n_sel - 1].s, w->cand[n_sel].s)"),
    "read-flags-not-shifted": lambda s: s.replace(
        "select_side(io->q + (size_t)t * dq, io->C1, io->C2, d, d->R, &w, rs, rw, NULL, 3);",
        "select_side(io->q + (size_t)t * dq, io->C1, io->C2, d, d->R, &w, rs, rw, NULL, 0);"),
    "half-flags-swapped": lambda s: s.replace(
        "flags |= 2 << flag_shift;", "flags |= 8 << flag_shift;").replace(
        "flags |= 4 << flag_shift;", "flags |= 2 << flag_shift;").replace(
        "flags |= 8 << flag_shift;", "flags |= 4 << flag_shift;"),
    "half-flag-wrong-pair": lambda s: s.replace(
        "near_tie(w->s64_1[w->h1[k - 1].id], w->s64_1[w->h1[k].id])",
        "near_tie(w->s64_1[w->h1[k > 1 ? k - 2 : 0].id], w->s64_1[w->h1[k - 1].id])"),
    "decay-weights-unnormalised": lambda s: s.replace(
        "  for (int j = 0; j < W; ++j) ww[j] /= z;\n", ""),
    "decay-softmax-router": lambda s: s.replace(
        "    ww[j] = 1.0 / (1.0 + exp(-(double)sw[j]));", "    ww[j] = exp((double)sw[j]);"),
    "decay-exponent-sign": lambda s: s.replace(
        "    const double dcy = exp(at * ww[j]);", "    const double dcy = exp(-at * ww[j]);"),
    "decay-toward-zero": lambda s: s.replace(
        "      row[col] = (float)(dcy * (double)row[col] + (1.0 - dcy) * (double)vt[col]);",
        "      row[col] = (float)(dcy * (double)row[col]);"),
    "decay-ignores-router": lambda s: s.replace(
        "    const double dcy = exp(at * ww[j]);", "    const double dcy = exp(at);"),
    "fp64-candidate-order": lambda s: s.replace(
        "float s = w->h1[a].s + w->h2[b].s;          /* float32 sum */",
        "float s = (float)(w->s64_1[w->h1[a].id] + w->s64_2[w->h2[b].id]);"),
}


@pytest.fixture(scope="module")
def mutant_dir():
    with tempfile.TemporaryDirectory(prefix="sdm_oracle_mut_") as d:
        yield d


def _caught_by_a_pin(pins_module, pin_names, so):
    """Run each pin on the broken build in a child process, in order, until one
    fails its assertion (True).  A pin whose child crashes does not count; the
    next pin is tried."""
    here = os.path.dirname(os.path.abspath(__file__))
    for pin in pin_names:
        code = ("import sys; sys.path[:0] = [%r, %r]\n"
                "import %s as m\n"
                "try:\n"
                "    m.%s(%r)\n"
                "except AssertionError:\n"
                "    sys.exit(17)\n") % (here, os.path.dirname(here), pins_module, pin, so)
        r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                           timeout=300)
        if r.returncode == 17:
            return True
    return False


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, mutant_dir):
    import pins
    with open(oracle.ORACLE_SRC) as f:
        src = f.read()
    bad = MUTANTS[name](src)
    assert bad != src, "mutation %s did not apply" % name
    c = os.path.join(mutant_dir, name + ".c")
    so = os.path.join(mutant_dir, name + ".so")
    with open(c, "w") as f:
        f.write(bad)
    oracle.compile_source(c, so)
    assert _caught_by_a_pin("pins", [p.__name__ for p in pins.ALL_PINS], so), \
        "no pin's assertion catches the mutation %r" % name
