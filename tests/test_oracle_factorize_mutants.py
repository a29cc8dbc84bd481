"""Plant plausible mistakes in copies of the factorisation reference and check the pins catch each.

Each mutant is oracle/factorize.py with one edit (a wrong or dropped sign,
a dropped factor, a multiplication where a solve belongs, a dropped dual
variable, the wrong singular pair, a stale factor, the wrong vector returned,
the keep rule removed), loaded as a separate module.  The pins of
test_oracle_factorize.py are run against it with the module swapped in; at
least one must fail.

Two edits are left out because they do not change what the reference computes
on the inputs it is given: starting R from Omega^T itself instead of its SVID
projection (a matrix of random signs with one magnitude is its own SVID
projection), and taking sign(0) as -1 (a convention of the packed layout that
only exact zeros reach).
"""
import inspect
import os
import types

import numpy as np
import pytest

import oracle
import test_oracle_factorize as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "factorize.py")

MUTANTS = {
    "dual_update_sign": ("Ud = Ud + L - Z", "Ud = Ud + Z - L"),
    "dual_dropped": ("Ud = Ud + L - Z", "Ud = Ud"),
    "rhs_dual_sign": ("rho * (Z - Ud)", "rho * (Z + Ud)"),
    "projection_without_dual": ("Z = svid_matrix(L + Ud)", "Z = svid_matrix(L)"),
    "rhs_drops_2": ("WR = 2.0 * W @ R.T", "WR = W @ R.T"),
    "gram_drops_2": ("G = 2.0 * R @ R.T + rho", "G = R @ R.T + rho"),
    "multiply_not_solve": ("L = np.linalg.solve(G, (WR + rho * (Z - Ud)).T).T", "L = (WR + rho * (Z - Ud)) @ G"),
    "svid_of_signed_matrix": ("np.linalg.svd(np.abs(M)", "np.linalg.svd(M"),
    "svid_second_pair": ("u = np.abs(U[:, 0]) * np.sqrt(sig[0])", "u = np.abs(U[:, 1]) * np.sqrt(sig[0])"),
    "right_step_uses_old_L": ("Rn = admm_left(W.T, Ln.T, R.T", "Rn = admm_left(W.T, L.T, R.T"),
    "returns_unprojected_L": ("    return Z\n", "    return L\n"),
    "mid_sum_not_product": ('"mid": mL * mR', '"mid": mL + mR'),
    "keeps_every_pass": ("if err < best:", "if True:"),
}


def _mutant(name):
    before, after = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(before) >= 1, f"mutant {name}: pattern not in the source"
    mod = types.ModuleType(f"factorize_{name}")
    exec(compile(src.replace(before, after, 1), f"factorize_{name}.py", "exec"), mod.__dict__)
    return mod


def _run_pin(fn, oracle_mod):
    params = inspect.signature(fn).parameters
    marks = getattr(fn, "pytestmark", [])
    cases = [m.args for m in marks if m.name == "parametrize"]
    if "oracle_mod" in params:
        fn(oracle_mod)
    elif cases:
        names, values = cases[0]
        names = [x.strip() for x in names.split(",")]
        for v in values:
            fn(**dict(zip(names, v if isinstance(v, tuple) else (v,))))
    else:
        fn()


def test_unmutated_reference_passes_every_pin(oracle_mod):
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if name.startswith("test_"):
            _run_pin(fn, oracle_mod)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, oracle_mod, monkeypatch):
    monkeypatch.setattr(pins, "F", _mutant(name))
    failed = []
    for pin, fn in inspect.getmembers(pins, inspect.isfunction):
        if not pin.startswith("test_"):
            continue
        try:
            with np.errstate(all="ignore"):
                _run_pin(fn, oracle_mod)
        except Exception:  # an assertion, or the mutant's arithmetic breaking down
            failed.append(pin)
    assert failed, f"mutant {name} passed every pin"
