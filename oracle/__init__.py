"""CPU oracle of the R-KV decode-time KV compression step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference leg of ``bench.py`` may import this package.  The
product library never loads it and has no CPU fallback.

Two independent formulations of the same definition:

* ``rkv_oracle.c``: plain nested loops in double precision, loaded through
  ctypes (``liboracle.so``, built by :func:`build`);
* ``rkv_oracle_np.py``: a vectorised NumPy float64 twin.

Both read the same bf16 bit patterns the GPU reads.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional

import numpy as np

from . import rkv_oracle_np as np_oracle  # noqa: F401  (re-exported)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rkv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib: Optional[ctypes.CDLL] = None

RED_MEAN, RED_MAX = 0, 1
POOL_MAX, POOL_MEAN = 0, 1


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (-O2, no fast-math, OpenMP over units)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, f64, i64 = ctypes.c_int, ctypes.c_double, ctypes.c_longlong
        _lib.rkv_oracle_importance.argtypes = [P, P, i32, i32, i32, i32, i32, P]
        _lib.rkv_oracle_inv_norm.argtypes = [P, i32, i32, P]
        _lib.rkv_oracle_redundancy.argtypes = [P, i32, i32, i32, i32, P]
        _lib.rkv_oracle_softmax.argtypes = [P, i32, P]
        _lib.rkv_oracle_joint.argtypes = [P, P, i32, f64, P]
        _lib.rkv_oracle_select.argtypes = [P, i32, i32, i32, P]
        _lib.rkv_oracle_shared_select.argtypes = [P, i32, i64, i32, i32, i32, P, P]
        _lib.rkv_oracle_compact.argtypes = [P, P, i32, i32, P]
        _lib.rkv_oracle_unit.argtypes = [P, P, i32, i32, i32, i32, i32, f64, i32, i32,
                                         P, P, P, P, P]
        _lib.rkv_oracle_units.argtypes = [i32, P, P, i64, P, P, P, i32, i32, i32, i32, i32,
                                          P, P, P, P, i64, P, i64, i32]
        for f in ("rkv_oracle_importance", "rkv_oracle_inv_norm", "rkv_oracle_redundancy",
                  "rkv_oracle_softmax", "rkv_oracle_joint", "rkv_oracle_select",
                  "rkv_oracle_compact", "rkv_oracle_unit", "rkv_oracle_units",
                  "rkv_oracle_shared_select"):
            getattr(_lib, f).restype = None
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _u16(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.uint16)


def importance(q_bits, k_bits, N: int, pool: int = POOL_MAX) -> np.ndarray:
    q = _u16(q_bits)
    k = _u16(k_bits)
    G, w, D = q.shape
    out = np.empty(N - w, dtype=np.float64)
    lib().rkv_oracle_importance(_ptr(q), _ptr(k), G, w, D, N, pool, _ptr(out))
    return out


def inv_norm(k_bits, N: int) -> np.ndarray:
    k = _u16(k_bits)
    out = np.empty(N, dtype=np.float64)
    lib().rkv_oracle_inv_norm(_ptr(k), N, k.shape[-1], _ptr(out))
    return out


def redundancy(k_bits, N: int, w: int, mode: int = RED_MEAN) -> np.ndarray:
    k = _u16(k_bits)
    out = np.empty(N - w, dtype=np.float64)
    lib().rkv_oracle_redundancy(_ptr(k), N, k.shape[-1], N - w, mode, _ptr(out))
    return out


def softmax(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty_like(x)
    lib().rkv_oracle_softmax(_ptr(x), x.shape[0], _ptr(out))
    return out


def joint(I, R, lam: float) -> np.ndarray:
    I = np.ascontiguousarray(I, dtype=np.float64)
    R = np.ascontiguousarray(R, dtype=np.float64)
    out = np.empty_like(I)
    lib().rkv_oracle_joint(_ptr(I), _ptr(R), I.shape[0], float(lam), _ptr(out))
    return out


def select(Z, N: int, budget: int) -> np.ndarray:
    Z = np.ascontiguousarray(Z, dtype=np.float64)
    out = np.empty(budget, dtype=np.int32)
    lib().rkv_oracle_select(_ptr(Z), Z.shape[0], N, budget, _ptr(out))
    return out


def compact(src_bits, kept) -> np.ndarray:
    src = _u16(src_bits)
    kept = np.ascontiguousarray(kept, dtype=np.int32)
    D = src.shape[-1]
    out = np.empty((kept.shape[0], D), dtype=np.uint16)
    lib().rkv_oracle_compact(_ptr(src), _ptr(kept), kept.shape[0], D, _ptr(out))
    return out


def unit(q_bits, k_bits, N: int, budget: int, lam: float, red_mode: int = RED_MEAN,
         pool: int = POOL_MAX) -> Dict[str, np.ndarray]:
    q = _u16(q_bits)
    k = _u16(k_bits)
    G, w, D = q.shape
    M = N - w
    out = {n: np.empty(M, dtype=np.float64) for n in ("I", "r", "R", "Z")}
    kept = np.empty(budget, dtype=np.int32)
    lib().rkv_oracle_unit(_ptr(q), _ptr(k), G, w, D, N, budget, float(lam), red_mode, pool,
                          _ptr(out["I"]), _ptr(out["r"]), _ptr(out["R"]), _ptr(out["Z"]),
                          _ptr(kept))
    out["kept"] = kept
    return out


def units(q_bits, k_bits, N, budget, lam, red_mode: int = RED_MEAN, pool: int = POOL_MAX,
          n_threads: int = 1) -> Dict[str, np.ndarray]:
    """Many units: q_bits [U, G, w, D], k_bits [U, rows, D]; N, budget, lam per unit.

    Returns I, r, R, Z as [U, rows] float64 (first N-w entries valid per unit)
    and kept as [U, max budget] int32 (first budget entries valid).
    """
    q = _u16(q_bits)
    k = _u16(k_bits)
    U, G, w, D = q.shape
    rows = k.shape[1]
    N = np.ascontiguousarray(np.broadcast_to(np.asarray(N, dtype=np.int32), (U,)))
    budget = np.ascontiguousarray(np.broadcast_to(np.asarray(budget, dtype=np.int32), (U,)))
    lam = np.ascontiguousarray(np.broadcast_to(np.asarray(lam, dtype=np.float64), (U,)))
    out = {n: np.zeros((U, rows), dtype=np.float64) for n in ("I", "r", "R", "Z")}
    bmax = int(budget.max())
    kept = np.zeros((U, bmax), dtype=np.int32)
    lib().rkv_oracle_units(U, _ptr(q), _ptr(k), rows * D, _ptr(N), _ptr(budget), _ptr(lam),
                           G, w, D, red_mode, pool, _ptr(out["I"]), _ptr(out["r"]),
                           _ptr(out["R"]), _ptr(out["Z"]), rows, _ptr(kept), bmax,
                           int(n_threads))
    out["kept"] = kept
    return out


def shared_select(Z_heads, N: int, budget: int):
    """Shared selection over the heads of one (sequence, layer): Z_heads [H, M]
    per-head joint scores of the M = N - w candidates.  Returns (Zsum [M],
    kept [budget]): the top budget - w candidates of the head sum plus the window."""
    Z = np.ascontiguousarray(Z_heads, dtype=np.float64)
    H, M = Z.shape
    out = np.empty(M, dtype=np.float64)
    kept = np.empty(budget, dtype=np.int32)
    lib().rkv_oracle_shared_select(_ptr(Z), H, M, M, N, budget, _ptr(out), _ptr(kept))
    return out, kept


def shared_units(q_bits, k_bits, N: int, budget: int, lam: float, red_mode: int = RED_MEAN,
                 pool: int = POOL_MAX, n_threads: int = 1) -> Dict[str, np.ndarray]:
    """The shared-selection step of one (sequence, layer): q_bits [H, G, w, D],
    k_bits [H, rows, D] (every head N rows).  Per-head I, r, R, Z as in `units`,
    plus Zsum [M] and the one kept set [budget] every head uses."""
    out = units(q_bits, k_bits, N, budget, lam, red_mode=red_mode, pool=pool, n_threads=n_threads)
    w = _u16(q_bits).shape[2]
    M = N - w
    out["Zsum"], out["kept_shared"] = shared_select(out["Z"][:, :M], N, budget)
    return out
