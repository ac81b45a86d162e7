"""Plant plausible mistakes in the numpy parts of the oracle (the compensator's
subspace iteration and split, the target and residual of the quantiser
rounds, the round selection, the kurtosis and the rank-budget split) and
check that the pins catch each one.

Each mutant edits one snippet of oracle/__init__.py, loads the edited source
as a separate module (on the CPU, in this process only) and runs the pins of
the quantiser and rank parts against it; at least one pin must fail.  The C
parts of the oracle have their own mutants (test_oracle_mutations.py).
"""
import os
import types

import pytest

import test_oracle_lorc_pins as lorc_pins
import test_oracle_rank_pins as rank_pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "__init__.py")

MUTANTS = {
    "split_unbalanced": ("""    U[:, :m] = (Y @ P) * root[None, :]
    V[:m] = (P.T @ B) * inv[:, None]""", """    U[:, :m] = (Y @ P) * (root * root)[None, :]
    V[:m] = (P.T @ B) * (inv * inv)[:, None]"""),
    "eigen_ascending": ("""    order = np.argsort(-lam, kind="stable")""", """    order = np.argsort(lam, kind="stable")"""),
    "rsvd_without_orthonormal_basis": ("""        Y = _orth(R @ _orth(R.T @ Y))""", """        Y = R @ (R.T @ Y)"""),
    "residual_sign": ("""    return (_f16(W_bits) - d).astype(np.float32)""", """    return (d - _f16(W_bits)).astype(np.float32)"""),
    "target_adds_compensator": ("""        T = (T - (U[:, p:p + 1] * V[p:p + 1, :]).astype(np.float32)).astype(np.float32)""",
                                """        T = (T + (U[:, p:p + 1] * V[p:p + 1, :]).astype(np.float32)).astype(np.float32)"""),
    "round_kept_is_worst": ("""        if best is None or errs[-1] < errs[best["round"]]:""",
                            """        if best is None or errs[-1] > errs[best["round"]]:"""),
    "kurtosis_uncentred": ("""    d = w - w.mean()""", """    d = w"""),
    "ranks_tie_to_lower_score": ("""    order = sorted(range(n), key=lambda i: (-frac[i], -s[i], i))""",
                                 """    order = sorted(range(n), key=lambda i: (-frac[i], s[i], i))"""),
    "ranks_negative_scores_by_magnitude": ("""    s = [max(float(x), 0.0) for x in scores]""",
                                           """    s = [abs(float(x)) for x in scores]"""),
    "ranks_budget_off_by_one": ("""    units = min(n * avg_rank // 8, cap * n)""", """    units = min(n * avg_rank // 8 + 1, cap * n)"""),
    "rsvd_no_power_iterations": ("""    for _ in range(power_iters):
        Y = _orth(R @ _orth(R.T @ Y))""", """    for _ in range(0):
        Y = _orth(R @ _orth(R.T @ Y))"""),
    "rounds_ignore_compensator": ("""        T = lorc_target(W, U16, V16)""", """        T = lorc_target(W)"""),
    "round_error_of_unrounded_pieces": ("""            E = R.astype(np.float64) - _f16(U16).astype(np.float64) @ _f16(V16).astype(np.float64)""",
                                        """            E = R.astype(np.float64) - U @ V"""),
    "kurtosis_over_m2": ("""    return float(np.mean(d ** 4)) / (m2 * m2) if m2 > 0 else 0.0""",
                         """    return float(np.mean(d ** 4)) / m2 if m2 > 0 else 0.0"""),
    "ranks_cap_not_refilled": ("""                left -= float(cap)
                changed = True""", """                left -= float(cap)"""),
}

PINS = [getattr(m, n) for m in (lorc_pins, rank_pins) for n in sorted(dir(m))
        if n.startswith("test_") and not n.startswith("test_hqq")]


def _mutated_module(old: str, new: str) -> types.ModuleType:
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found once: {old[:60]!r}"
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = SRC
    exec(compile(src.replace(old, new), SRC, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_python_mutant_is_caught(name, monkeypatch):
    mutant = _mutated_module(*MUTANTS[name])
    monkeypatch.setattr(lorc_pins, "oracle", mutant)
    monkeypatch.setattr(rank_pins, "oracle", mutant)
    failed = []
    for pin in PINS:
        try:
            pin()
        except Exception:                      # an AssertionError, or the mistake breaking a shape
            failed.append(pin.__name__)
    assert failed, f"mutant {name} survived every pin"


def test_unmutated_oracle_passes_every_pin(monkeypatch):
    """The same harness with no edit: every pin passes (so a caught mutant is
    caught because of its edit)."""
    clean = _mutated_module("import numpy as np", "import numpy as np")
    monkeypatch.setattr(lorc_pins, "oracle", clean)
    monkeypatch.setattr(rank_pins, "oracle", clean)
    for pin in PINS:
        pin()
