"""Parity measured at the granularity a kernel goes wrong at.

A defect confined to one 128-row tile, one ring slot or one chunk boundary
is diluted in a rel-Frobenius taken over the whole output: in an 8k head a
tile is 1/64 of the rows, so a tile that is 15% wrong moves the whole-output
figure by about 2%.  `worst_rel` therefore reports the largest rel-Frobenius
error over the whole array, over each (batch, head) slice and over each
128-row tile of each (batch, head) matrix, and the tests hold that worst
value to the same tolerance as the whole.

Layouts: [..., rows, cols] arrays of rank >= 4 are (batch, head) matrices
(outputs [B,H,N,d], states [B,H,d_k,d_v]); rank 3 is one row per (batch,
head) (decode outputs [B,H,d]); rank 2 is one matrix; rank <= 1 is checked
whole.

Test infrastructure: it calls the oracle's rel_frobenius for the whole
array and restates the same quotient per block.
"""
from __future__ import annotations

import numpy as np

import oracle

TILE = 128


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def _quot(num2, den2):
    """sqrt(num2 / den2) elementwise, with 0/0 = 0 and x/0 = inf."""
    num2, den2 = np.asarray(num2, np.float64), np.asarray(den2, np.float64)
    out = np.zeros(np.broadcast(num2, den2).shape)
    pos = den2 > 0
    out[pos] = np.sqrt(num2[pos] / den2[pos])
    out[~pos & (num2 > 0)] = np.inf
    return out


def blocks(x, ref, tile=TILE):
    """[(where, rel-Frobenius error)] for the whole array, each (batch, head)
    and each `tile`-row block."""
    x, ref = _f64(x), _f64(ref)
    if x.shape != ref.shape:
        raise ValueError(f"shape {x.shape} against reference {ref.shape}")
    out = [("whole", oracle.rel_frobenius(x, ref))]
    if x.ndim <= 1:
        return out
    if x.ndim == 3:  # one row per (batch, head)
        d2 = ((x - ref) ** 2).sum(-1)
        r2 = (ref ** 2).sum(-1)
        for idx, e in np.ndenumerate(_quot(d2, r2)):
            out.append((f"(b,h)={tuple(int(i) for i in idx)}", float(e)))
        return out
    lead = x.shape[:-2] if x.ndim >= 4 else (1,)
    rows = x.shape[-2]
    d2 = ((x - ref) ** 2).sum(-1).reshape(-1, rows)   # [units, rows]
    r2 = (ref ** 2).sum(-1).reshape(-1, rows)
    unit = _quot(d2.sum(-1), r2.sum(-1))
    starts = np.arange(0, rows, tile) if rows else np.zeros(0, dtype=int)
    if rows:
        td = np.add.reduceat(d2, starts, axis=1)
        tr = np.add.reduceat(r2, starts, axis=1)
        tiles = _quot(td, tr)
    for u in range(d2.shape[0]):
        name = (f"(b,h)={tuple(int(i) for i in np.unravel_index(u, lead))}" if x.ndim >= 4
                else "matrix")
        out.append((name, float(unit[u])))
        if rows and len(starts) > 1:
            for t, r0 in enumerate(starts):
                out.append((f"{name} rows {r0}:{min(r0 + tile, rows)}", float(tiles[u, t])))
    return out


def worst(x, ref, tile=TILE):
    """(where, error) of the worst block."""
    return max(blocks(x, ref, tile), key=lambda b: (np.isnan(b[1]), b[1]))


class WorstError(float):
    """A rel-Frobenius error that also says where it was found (shown when an
    assertion on it fails)."""

    def __new__(cls, value, where):
        obj = super().__new__(cls, value)
        obj.where = where
        return obj

    def __repr__(self):
        return f"{float(self):.4g} (worst at {self.where})"


def worst_rel(x, ref, tile=TILE) -> float:
    """The largest rel-Frobenius error over the whole array, each (batch,
    head) and each `tile`-row block (NaN counts as the worst)."""
    where, e = worst(x, ref, tile)
    return WorstError(float("inf") if np.isnan(e) else e, where)
