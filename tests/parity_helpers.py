"""Shared comparison helpers for the GPU parity tests (no method arithmetic:
every expected value still comes from ``oracle``)."""
from __future__ import annotations

import itertools

import numpy as np

import oracle

BF16_ULP_TOL = 1


def bf16_ordered(bits: np.ndarray) -> np.ndarray:
    """Map bf16 bit patterns to integers whose differences count ulps."""
    b = bits.astype(np.int32)
    return np.where(b & 0x8000, 0x8000 - b, b)


def assert_bf16_close(got_bits: np.ndarray, ref_bits: np.ndarray, tol: int = BF16_ULP_TOL):
    d = np.abs(bf16_ordered(got_bits) - bf16_ordered(ref_bits))
    assert d.max(initial=0) <= tol, \
        f"max bf16 ulp distance {d.max()} at {np.unravel_index(d.argmax(), d.shape)}"


def tile_rows(M: int, tile: int = 256) -> np.ndarray:
    """One row in every `tile`-row M-tile, its position inside the tile
    varying from tile to tile, plus the first, the last and the tile edges
    around the middle."""
    rows = {(t * tile + (t * 97 + 13) % tile) for t in range((M + tile - 1) // tile)}
    mid = (M // 2) // tile * tile
    rows |= {0, 1, M - 2, M - 1, mid - 1, mid, tile - 1, tile}
    return np.array(sorted(r for r in rows if 0 <= r < M), np.int64)


def assert_codes_admissible(Qx: np.ndarray, s_x: np.ndarray, Y: np.ndarray, Ya: np.ndarray,
                            max_flags: int = 10):
    """The quantiser's codes and row scales for normalised rows whose exact
    values admit two bf16 neighbours at a few elements (Y vs Ya): every row
    must equal the oracle's codes and scale of Y's row with some choice of
    Y or Ya at each such element (the rows without such elements: Y's)."""
    Y = np.ascontiguousarray(Y)
    rq, rs = oracle.quantize_rows_bf16(Y, rotate=True)
    flagged_rows = np.nonzero((Y != Ya).any(axis=1))[0]
    plain = np.ones(Y.shape[0], bool)
    plain[flagged_rows] = False
    assert np.array_equal(Qx[plain], rq[plain])
    assert np.array_equal(s_x[plain].view(np.uint32), rs[plain].view(np.uint32))
    for m in flagged_rows:
        idx = np.nonzero(Y[m] != Ya[m])[0]
        assert idx.size <= max_flags, f"row {m}: {idx.size} elements near a midpoint"
        variants = np.repeat(Y[m][None, :], 2 ** idx.size, axis=0)
        for v, choice in enumerate(itertools.product((0, 1), repeat=idx.size)):
            pick = np.array(choice, bool)
            variants[v, idx[pick]] = Ya[m, idx[pick]]
        vq, vs = oracle.quantize_rows_bf16(variants, rotate=True)
        ok = (vq == Qx[m][None, :]).all(axis=1) & (vs.view(np.uint32) == s_x[m].view(np.uint32))
        assert ok.any(), f"row {m}: codes match no admissible rounding of its normalised values"
