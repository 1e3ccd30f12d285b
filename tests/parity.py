"""Tolerance checks shared by the GPU parity tests.

A device value d matches the oracle value v when |d - v| <= 1e-3 * S + 1e-5
element by element, S being the oracle's error scale (the sum of absolute
terms behind v, propagated through the later steps), and the relative L2
error ||d - v|| / ||v|| is at most 2e-3.
"""
import concurrent.futures
import os

import numpy as np

REL = 1e-3
ABS = 1e-5
REL_L2 = 2e-3


def check(d, v, S, what: str, rel_l2: bool = True):
    d = np.asarray(d, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    S = np.asarray(S, dtype=np.float64)
    assert d.shape == v.shape, (what, d.shape, v.shape)
    assert np.all(np.isfinite(d)), f"{what}: non-finite device values"
    err = np.abs(d - v)
    tol = REL * S + ABS
    bad = err > tol
    if bad.any():
        i = int(np.argmax(err - tol))
        raise AssertionError(f"{what}: {int(bad.sum())}/{bad.size} outside tolerance; worst at {i}: "
                             f"device {d.flat[i]!r} oracle {v.flat[i]!r} tol {tol.flat[i]!r}")
    if rel_l2:
        nv = np.linalg.norm(v)
        if nv > 0:
            r = np.linalg.norm(d - v) / nv
            assert r <= REL_L2, f"{what}: relative L2 {r:.3g} > {REL_L2}"
    return float((err / tol).max()) if err.size else 0.0


def pmap(fn, items):
    """Runs fn over items on host threads (the oracle's C calls release the
    interpreter lock) and re-raises the first failure."""
    items = list(items)
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 4)) as ex:
        return list(ex.map(fn, items))
