"""The LB-ADMM oracle against its pins (CPU only), and each planted mistake caught."""
import importlib.util
import os

import numpy as np
import pytest

import admm_pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "admm.py")


def _module(source: str, name: str):
    spec = importlib.util.spec_from_loader(name, loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(source, SRC, "exec"), mod.__dict__)
    return mod


@pytest.fixture(scope="module")
def adm():
    from oracle import admm

    return admm


@pytest.mark.parametrize("pin", admm_pins.ALL, ids=lambda f: f.__name__)
def test_admm_oracle_pin(adm, pin):
    pin(adm)


# Plausible mistakes, each planted in a copy of the oracle's source: (name, original, replacement).
MUTANTS = [
    ("no dual update", 'LA = st["LA"] + A - ZA', 'LA = st["LA"]'),
    ("dual with the wrong sign", 'project(A + st["LA"])', 'project(A - st["LA"])'),
    ("scale = max instead of mean", "np.abs(M).sum(axis=1) / M.shape[1]", "np.abs(M).max(axis=1)"),
    ("sign(0) = -1", "np.where(M >= 0.0, 1, -1)", "np.where(M > 0.0, 1, -1)"),
    ("least squares without the penalty target", "R = W @ F + rho * C", "R = W @ F"),
    ("least squares without the penalty diagonal", "H = F.T @ F + rho * np.eye(r)", "H = F.T @ F"),
    ("B update from the previous A", 'B = ls_update(W.T, A,', 'B = ls_update(W.T, st["A"],'),
    ("penalty scaled by the updated factor", 'penalty(st["B"], lam)', 'penalty(st["A"], lam)'),
    ("penalty without 1/r", "return lam * float(np.sum(F * F)) / F.shape[1]", "return lam * float(np.sum(F * F))"),
    ("balance the wrong way", "c = np.sqrt(rB / rA)", "c = np.sqrt(rA / rB)"),
    ("Cholesky-QR with L^T", "return np.linalg.solve(L, Y.T).T", "return np.linalg.solve(L.T, Y.T).T"),
    ("column balance without the square root", "c = np.sqrt(np.linalg.norm(B, axis=0) / np.linalg.norm(A, axis=0))",
     "c = np.linalg.norm(B, axis=0) / np.linalg.norm(A, axis=0)"),
    ("result from the latent factor", 'out = (st["SA"].copy(), st["SB"].copy(), s1, s2)',
     'out = (st["SA"].copy(), st["SB"].copy(), st["sA"], s2)'),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_admm_mutant_is_caught(name, old, new):
    with open(SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation site not found once: {old!r}"
    mutant = _module(src.replace(old, new), "admm_mutant")
    failed = []
    for pin in admm_pins.ALL:
        try:
            with np.errstate(all="ignore"):  # a broken mutant may overflow on its way to failing
                pin(mutant)
        except Exception as e:  # an assertion, or the mutant breaking outright
            failed.append((pin.__name__, type(e).__name__))
    assert failed, f"planted mistake not caught by any pin: {name}"
