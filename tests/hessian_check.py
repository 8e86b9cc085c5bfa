"""Per-block parity check of a GPU Hessian against the float64 oracle.

A Hessian from calibration data with outlier channels is dominated by a few
large diagonal entries (an outlier column scaled by 20 has H_ii near 400,
while a typical off-diagonal entry is near 1/sqrt(n)).  One Frobenius ratio
pooled over the whole sample therefore cannot see a wrong or misplaced
off-diagonal tile.  Here every sampled block is judged on its own: its
relative Frobenius error must stay within the tolerance (1e-3), so a block
holding another block's values (a transposed, shifted or swapped tile) fails
with an error near 1.

The sample covers, for a C x C Hessian computed in 256 x 256 tiles:
  * every 32 x 32 diagonal block;
  * one seeded 32 x 32 block inside every upper-triangle 256 x 256 tile
    (I <= J), on or above the diagonal, so every tile the kernel computes is
    looked at;
  * seeded random 128 x 128 tiles at 32-aligned offsets anywhere in H (upper
    and lower triangle, some straddling the 256-tile boundaries).
"""
from __future__ import annotations

import numpy as np

TOL = 1e-3
TILE = 256


def tile_blocks(C: int, rng: np.random.Generator, tile: int = TILE):
    """(r0, c0) of one 32 x 32 block inside every upper-triangle tile, plus every diagonal block."""
    nb = (C + tile - 1) // tile
    out = [(32 * g, 32 * g) for g in range(C // 32)]
    for I in range(nb):
        for J in range(I, nb):
            rows = [r for r in range(I * tile, min(C, (I + 1) * tile), 32)]
            cols = [c for c in range(J * tile, min(C, (J + 1) * tile), 32)]
            cand = [(r, c) for r in rows for c in cols if c >= r]
            out.append(cand[int(rng.integers(0, len(cand)))])
    return out


def random_tiles(C: int, rng: np.random.Generator, count: int, b: int = 128):
    """(r0, c0) of `count` b x b tiles at 32-aligned offsets (anywhere, both triangles)."""
    hi = (C - b) // 32 + 1
    return [(32 * int(rng.integers(0, hi)), 32 * int(rng.integers(0, hi))) for _ in range(count)]


def block_errors(Hg: np.ndarray, refs: np.ndarray, starts, b: int) -> np.ndarray:
    """Relative Frobenius error of each b x b block Hg[r0:r0+b, c0:c0+b] against refs[m]."""
    errs = np.empty(len(starts))
    for m, (r0, c0) in enumerate(starts):
        got = Hg[r0:r0 + b, c0:c0 + b].astype(np.float64)
        ref = refs[m]
        den = float(np.linalg.norm(ref))
        num = float(np.linalg.norm(got - ref))
        errs[m] = (num / den) if den > 0 else (0.0 if num == 0 else np.inf)
    return errs


def check_blocks(Hg: np.ndarray, refs: np.ndarray, starts, b: int, tol: float = TOL):
    """Asserts every block's relative Frobenius error is within tol; reports the worst blocks."""
    errs = block_errors(Hg, refs, starts, b)
    bad = np.flatnonzero(~(errs <= tol))
    assert bad.size == 0, (f"{bad.size} of {len(starts)} {b}x{b} blocks above {tol}: " +
                           ", ".join(f"({starts[i][0]},{starts[i][1]}): {errs[i]:.3g}" for i in bad[:8]))
    return float(errs.max()) if len(errs) else 0.0


def check_hessian(Hg: np.ndarray, Xb: np.ndarray, oracle_mod, rng: np.random.Generator,
                  n_random: int = 64, every_tile: bool = True, tile_sample: int | None = None):
    """Full per-block check of a GPU Hessian Hg (float32 [C, C]) of bf16 X (uint16 bits).

    every_tile: one block in every upper-triangle 256 x 256 tile; otherwise `tile_sample`
    seeded tiles.  Returns the largest relative error seen."""
    C = Xb.shape[1]
    starts = tile_blocks(C, rng)
    if not every_tile:
        diag = starts[:C // 32]
        rest = starts[C // 32:]
        pick = rng.choice(len(rest), size=min(tile_sample or 0, len(rest)), replace=False)
        starts = diag + [rest[int(i)] for i in sorted(pick)]
    worst = check_blocks(Hg, oracle_mod.hessian_blocks(Xb, [s[0] for s in starts], [s[1] for s in starts], 32),
                         starts, 32)
    if n_random and C >= 128:
        tiles = random_tiles(C, rng, n_random)
        worst = max(worst, check_blocks(
            Hg, oracle_mod.hessian_blocks(Xb, [t[0] for t in tiles], [t[1] for t in tiles], 128), tiles, 128))
    return worst
