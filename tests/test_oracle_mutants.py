"""The pins have teeth: plausible slips planted in a copy of the NumPy oracle
(on the CPU, never in the product) each fail at least one pin."""
import inspect
import types

import pytest

import oracle
from oracle import rkv_oracle_np
from tests import test_oracle_pins as pins

MUTANTS = {
    "logit scale dropped": ("/ np.sqrt(D)", ""),
    "causal mask dropped": ("logits = np.where(visible[None], logits, -np.inf)", "pass"),
    "GQA mean instead of max": ("ihat = a.max(axis=0) if pool == POOL_MAX else a.mean(axis=0)",
                                "ihat = a.mean(axis=0)"),
    "I not renormalised": ("return ihat / ihat.sum()", "return ihat"),
    "diagonal kept in similarity": ("off = ~np.eye(N, dtype=bool)",
                                    "off = np.ones((N, N), dtype=bool)"),
    "divisor N instead of N-1": ("[:M].sum(axis=1) / (N - 1)", "[:M].sum(axis=1) / N"),
    "window keys left out of r": ("C = kh @ kh.T", "C = kh @ kh.T; C[:, M:] = 0.0"),
    "keys not normalised": ("kh = k * inv_norm(k_bits, N)[:, None]\n    C", "kh = k\n    C"),
    "sign of R flipped": ("return lam * I - (1.0 - lam) * R", "return lam * I + (1.0 - lam) * R"),
    "lambda on the wrong term": ("return lam * I - (1.0 - lam) * R",
                                 "return (1.0 - lam) * I - lam * R"),
    "ties keep the highest index": ("order = np.lexsort((np.arange(M), -Z))",
                                    "order = np.lexsort((-np.arange(M), -Z))"),
}


def _mutant(old, new):
    src = inspect.getsource(rkv_oracle_np)
    assert old in src
    mod = types.ModuleType("rkv_oracle_np_mutant")
    exec(compile(src.replace(old, new, 1), "<mutant>", "exec"), mod.__dict__)
    return mod


def _numpy_pin_calls():
    """(name, callable) for every pin that accepts the NumPy twin."""
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        params = inspect.signature(fn).parameters
        if "impl" not in params:
            continue
        kwargs_list = [{}]
        if "mode" in params:
            kwargs_list = [dict(k, mode=m) for k in kwargs_list
                           for m in (oracle.RED_MEAN, oracle.RED_MAX)]
        if "seed" in params:
            kwargs_list = [dict(k, seed=s) for k in kwargs_list for s in range(6)]
        for kw in kwargs_list:
            calls.append((name, fn, kw))
    return calls


@pytest.mark.parametrize("mutation", list(MUTANTS))
def test_planted_mistake_fails_a_pin(mutation, monkeypatch):
    monkeypatch.setitem(pins.IMPLS, "numpy", _mutant(*MUTANTS[mutation]))
    failed = []
    for name, fn, kw in _numpy_pin_calls():
        try:
            fn(impl="numpy", **kw)
        except AssertionError:
            failed.append(name)
    assert failed, f"no pin caught: {mutation}"


def test_unmutated_twin_passes_every_pin():
    for name, fn, kw in _numpy_pin_calls():
        fn(impl="numpy", **kw)
