"""Tile-local parity checks and row sampling for the full-size workloads.

A whole-tensor relative Frobenius error dilutes a local fault: the LoRA term
is a few percent of Y and dX, so one 256 x 256 output tile that dropped it
moves the whole-tensor error by ~0.2 %, far inside 1e-2.  These helpers check
the same bar tile by tile:

* ``rows_every_tile``: token rows to compare -- ``per_tile`` seeded rows from
  every ``tile``-row band (the GEMM's CTA token tile is 256), plus the first and
  the last (ragged) row.
* ``tile_errors``: the relative Frobenius error of every (row band x column
  band) tile of a sampled [rows, C] result against the oracle's rows.
* ``block_errors``: the same over the 16 x 16 blocks of a full [R, C] result
  (dA, dB), skipping blocks whose reference is exactly zero.

The checks need no GPU; ``tests/test_parity_tiles.py`` shows on the CPU that a
result with one tile wrong fails them while its whole-tensor error passes.
"""
from __future__ import annotations

import numpy as np


def rows_every_tile(M: int, seed: int, tile: int = 256, per_tile: int = 1) -> np.ndarray:
    """Sorted unique row indices: ``per_tile`` random rows of every band of
    ``tile`` rows, plus rows 0 and M - 1."""
    g = np.random.default_rng(seed)
    rows = [0, M - 1]
    for t0 in range(0, M, tile):
        t1 = min(M, t0 + tile)
        rows.extend(int(v) for v in g.choice(np.arange(t0, t1), size=min(per_tile, t1 - t0), replace=False))
    return np.unique(np.asarray(rows, np.int64))


def _relfro(got, ref):
    d = np.linalg.norm(got - ref)
    n = np.linalg.norm(ref)
    return d / n if n > 0 else d


def tile_errors(got, ref, rows, row_tile: int = 256, col_tile: int = 256):
    """{(row band, column band): relative Frobenius error} over the sampled
    rows.  got, ref: [len(rows), C]; rows: the token index of each row."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rows = np.asarray(rows, np.int64)
    assert got.shape == ref.shape and got.shape[0] == rows.shape[0]
    C = got.shape[1]
    band = rows // row_tile
    out = {}
    for b in np.unique(band):
        sel = band == b
        for c0 in range(0, C, col_tile):
            g = got[sel, c0:c0 + col_tile]
            r = ref[sel, c0:c0 + col_tile]
            out[(int(b), c0 // col_tile)] = _relfro(g, r)
    return out


def block_errors(got, ref, block: int = 16):
    """{(i, j): relative Frobenius error} of every block x block block of a
    full result whose reference block is not exactly zero."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape
    R, C = ref.shape
    out = {}
    for i0 in range(0, R, block):
        for j0 in range(0, C, block):
            r = ref[i0:i0 + block, j0:j0 + block]
            if not np.any(r):
                continue
            out[(i0 // block, j0 // block)] = _relfro(got[i0:i0 + block, j0:j0 + block], r)
    return out


def worst(errs: dict):
    """(key, error) of the largest error; (None, 0.0) when there is none."""
    if not errs:
        return None, 0.0
    k = max(errs, key=errs.get)
    return k, errs[k]


def assert_tiles(name, got, ref, rows, tol, row_tile=256, col_tile=256):
    k, e = worst(tile_errors(got, ref, rows, row_tile, col_tile))
    assert e <= tol, f"{name}: tile {k} (row band, column band) rel err {e:.3e} > {tol}"
    return e


def assert_blocks(name, got, ref, tol, block=16):
    k, e = worst(block_errors(got, ref, block))
    assert e <= tol, f"{name}: block {k} rel err {e:.3e} > {tol}"
    return e
