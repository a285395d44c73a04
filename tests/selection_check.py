"""Validity of a CS4A block selection judged on the kernel's own pooled masses.

Where the oracle's decision sits within its margin of a flip (two masses or a
running sum within 1e-4 of each other or of the threshold), several selections
are correct, and the GPU's list is checked to be one of them instead of being
compared bit for bit.  The rules follow the selection the SparVAR pages describe
("SparVAR", ai.info summary, "Methodology in Plain English", CS4A paragraph:
the most important key blocks by pooled attention mass) under the workload's
mass-threshold reading (the smallest set whose mass reaches the threshold) and
the Top-K reading (a fixed number of the heaviest blocks):

mass threshold tau:
  (i)   heaviest first: every kept mass >= every dropped mass - tol;
  (ii)  minimal: the kept sum minus the smallest kept mass < tau + tol, unless a
        single block is kept;
  (iii) enough: the kept sum >= tau - tol, unless every block is kept.
Top-K with k blocks:
  exactly k blocks, and (i).
Both: the list is ascending, without repeats, inside [0, NKB), padded with -1.
"""
from __future__ import annotations

import numpy as np

TOL = 1e-5


def _list_ok(cnt, row, nkb):
    kept = np.asarray(row[:cnt])
    if cnt < 0 or cnt > nkb:
        return None, f"count {cnt} outside [0, {nkb}]"
    if kept.size and (kept.min() < 0 or kept.max() >= nkb):
        return None, "index outside [0, NKB)"
    if np.any(np.diff(kept) <= 0):
        return None, "list not strictly ascending"
    if np.any(np.asarray(row[cnt:]) != -1):
        return None, "tail not padded with -1"
    return kept, ""


def mass_selection_error(cnt, row, masses, tau, tol=TOL):
    """'' when (cnt, row) is a valid mass-threshold selection of ``masses``, else why not."""
    masses = np.asarray(masses, dtype=np.float64)
    nkb = masses.size
    kept, why = _list_ok(int(cnt), row, nkb)
    if kept is None:
        return why
    if kept.size == 0:
        return "empty selection"
    dropped = np.setdiff1d(np.arange(nkb), kept)
    mk = masses[kept]
    if dropped.size and mk.min() < masses[dropped].max() - tol:
        return "not heaviest first"
    total = mk.sum()
    if kept.size > 1 and total - mk.min() >= tau + tol:
        return "not minimal: the lightest kept block is not needed"
    if dropped.size and total < tau - tol:
        return "kept mass below the threshold"
    return ""


def topk_selection_error(cnt, row, masses, k, tol=TOL):
    """'' when (cnt, row) keeps exactly k of the heaviest ``masses``, else why not."""
    masses = np.asarray(masses, dtype=np.float64)
    nkb = masses.size
    if int(cnt) != k:
        return f"count {cnt}, expected {k}"
    kept, why = _list_ok(int(cnt), row, nkb)
    if kept is None:
        return why
    dropped = np.setdiff1d(np.arange(nkb), kept)
    if dropped.size and masses[kept].min() < masses[dropped].max() - tol:
        return "not heaviest first"
    return ""
