"""The dense GDN oracle against its pins (tests/gdn_pins.py), and plausible
mistakes planted in copies of it (on the CPU) that each pin set must catch."""
import os
import subprocess
import sys
import tempfile

import pytest

import gdn_pins
import oracle


@pytest.mark.parametrize("pin", gdn_pins.GDN_PINS, ids=lambda f: f.__name__)
def test_gdn_oracle_pin(pin):
    pin(None)


GDN_MUTANTS = {
    "prediction-from-ungated-state": lambda s: s.replace(
        "        s[j] = a * s[j];\n        pred += s[j] * (double)kt[j];",
        "        pred += s[j] * (double)kt[j];\n        s[j] = a * s[j];"),
    "forget-gate-dropped": lambda s: s.replace("        s[j] = a * s[j];\n", ""),
    "delta-sign-flipped": lambda s: s.replace(
        "for (int j = 0; j < dk; ++j) s[j] += e * (double)kt[j];",
        "for (int j = 0; j < dk; ++j) s[j] -= e * (double)kt[j];"),
    "beta-dropped": lambda s: s.replace(
        "const double e = b * ((double)vt[i] - pred);", "const double e = ((double)vt[i] - pred);"),
    "update-along-query": lambda s: s.replace(
        "for (int j = 0; j < dk; ++j) s[j] += e * (double)kt[j];",
        "for (int j = 0; j < dk; ++j) s[j] += e * (double)qt[j];"),
    "read-with-key": lambda s: s.replace(
        "for (int j = 0; j < dk; ++j) o += s[j] * (double)qt[j];",
        "for (int j = 0; j < dk; ++j) o += s[j] * (double)kt[j];"),
    "read-before-write": lambda s: s.replace(
        "      double pred = 0.0;\n",
        "      double o0 = 0.0;\n      for (int j = 0; j < dk; ++j) o0 += a * s[j] * (double)qt[j];\n"
        "      double pred = 0.0;\n").replace(
        "      if (J->o) J->o[(tq + t) * dv + i] = (float)o;",
        "      (void)o;\n      if (J->o) J->o[(tq + t) * dv + i] = (float)o0;"),
}


@pytest.fixture(scope="module")
def mutant_dir():
    with tempfile.TemporaryDirectory(prefix="gdn_oracle_mut_") as d:
        yield d


@pytest.mark.parametrize("name", sorted(GDN_MUTANTS))
def test_gdn_mutant_is_caught(name, mutant_dir):
    from test_oracle_mutations import _caught_by_a_pin
    with open(oracle.GDN_SRC) as f:
        src = f.read()
    bad = GDN_MUTANTS[name](src)
    assert bad != src, "mutation %s did not apply" % name
    c = os.path.join(mutant_dir, name + ".c")
    so = os.path.join(mutant_dir, name + ".so")
    with open(c, "w") as f:
        f.write(bad)
    oracle.compile_source(c, so)
    assert _caught_by_a_pin("gdn_pins", [p.__name__ for p in gdn_pins.GDN_PINS], so), \
        "no pin's assertion catches the mutation %r" % name
