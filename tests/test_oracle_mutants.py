"""The oracle pins must catch plausible mistakes.

Each case copies the oracle's C source, plants one mistake (a dropped gate, a
wrong sign, a wrong index, a wrong decay, a dropped scale), compiles it to a
temporary library and runs the pin tests against it with the real library
swapped out.  At least one pin must fail for every mutant.  Mistakes are
planted on the CPU only.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn2_oracle.c")

MUTANTS = {
    "erase gate dropped": ("e[c] = bt[c] * kt[c];", "e[c] = kt[c];"),
    "write gate dropped": ("z[j] = wt[j] * vt[j];", "z[j] = vt[j];"),
    "correction sign flipped": ("row[j] += kc * (z[j] - r[j]);", "row[j] += kc * (z[j] + r[j]);"),
    "decay halved": ("const double a = exp(lat[c]);", "const double a = exp(0.5 * lat[c]);"),
    "scale dropped": ("for (int j = 0; j < dv; ++j) ot[j] *= J->scale;", "for (int j = 0; j < dv; ++j) ot[j] *= 1.0;"),
    "erase gate read from head 0": ("const double* bt = J->b + ((size_t)t * H + h) * dk;",
                                    "const double* bt = J->b + ((size_t)t * H) * dk;"),
    "erase uses the query": ("e[c] = bt[c] * kt[c];", "e[c] = bt[c] * qt[c];"),
    "erase gate clamped to [0, 1]": ("e[c] = bt[c] * kt[c];", "e[c] = fmin(bt[c], 1.0) * kt[c];"),
}

PIN_TESTS = [
    pins.test_reduction_to_kda,
    pins.test_reduction_to_gated_deltanet,
    pins.test_reduction_to_deltanet,
    pins.test_delta_rule_overwrite_invariant,
    pins.test_full_range_erase_repeated_token_is_identity,
    pins.test_no_erase_is_decayed_linear_attention,
    pins.test_no_erase_no_write_is_pure_decay,
    pins.test_basis_keys_exact_example,
]


def _compile(tmp_path, src_text, name):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(src_text)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-pthread", str(c), "-o", str(so), "-lm"],
                   check=True)
    return str(so)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path, monkeypatch):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site not found: {old}"
    so = _compile(tmp_path, src.replace(old, new, 1), name.replace(" ", "_"))
    real = oracle._load()
    lib = ctypes.CDLL(so)
    for fn in ("oracle_gdn2_recurrent_f64", "oracle_kda_f64", "oracle_gdn_f64", "oracle_deltanet_f64"):
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
        getattr(lib, fn).restype = ctypes.c_int
    monkeypatch.setattr(oracle, "_lib", lib)
    failed = []
    for t in PIN_TESTS:
        try:
            t()
        except AssertionError:
            failed.append(t.__name__)
    assert failed, f"no pin caught mutant '{name}'"
