"""Comparison rules for the GPU-vs-oracle parity tests.

Codes must be bit-identical, except that a code may be the adjacent one where
the oracle's pre-rounding value lies within 2^-20 (relative) of a rounding
midpoint.  NaN codes compare by class (0x7F and 0xFF are both NaN).  Scales,
amax and global scales must be bit-identical (compared as raw bits).
"""
from __future__ import annotations

import numpy as np

from _exact import e2m1_grid, e4m3_grid

WINDOW = 2.0 ** -20
# Inside the 2^-20 window only a vanishing fraction of values can differ; a
# larger count is a systematic fault and fails at once.
MAX_WINDOW_CASES = 10000


def _mids(values):
    v = np.array([float(x) for x in values], dtype=np.float64)
    return (v[:-1] + v[1:]) / 2


E4_CODES, E4_VALS = e4m3_grid()
E2_CODES, E2_VALS = e2m1_grid()
E4_MIDS = _mids(E4_VALS)
E2_MIDS = _mids(E2_VALS)
E4_RANK = {c: i for i, c in enumerate(E4_CODES)}
E2_RANK = {c: i for i, c in enumerate(E2_CODES)}


def near_mid(pre: np.ndarray, mids: np.ndarray) -> np.ndarray:
    a = np.abs(pre.astype(np.float64))
    i = np.clip(np.searchsorted(mids, a), 1, len(mids) - 1)
    d = np.minimum(np.abs(a - mids[i - 1]), np.abs(a - mids[i]))
    return d <= WINDOW * a


def assert_bits_equal(got, want, what: str) -> None:
    g = np.ascontiguousarray(got)
    w = np.ascontiguousarray(want)
    assert g.shape == w.shape, (what, g.shape, w.shape)
    gb = g.view(np.uint32) if g.dtype == np.float32 else g
    wb = w.view(np.uint32) if w.dtype == np.float32 else w
    bad = np.flatnonzero(gb.reshape(-1) != wb.reshape(-1))
    assert bad.size == 0, f"{what}: {bad.size} mismatches, first at {bad[:5]}: got {g.reshape(-1)[bad[:5]]} " \
                          f"want {w.reshape(-1)[bad[:5]]}"


def fp8_mismatches(got: np.ndarray, want: np.ndarray) -> np.ndarray:
    """Indices where the E4M3 codes differ, NaN codes counted as equal."""
    g = got.reshape(-1)
    w = want.reshape(-1)
    nan_g = (g & 0x7F) == 0x7F
    nan_w = (w & 0x7F) == 0x7F
    return np.flatnonzero((g != w) & ~(nan_g & nan_w))


def assert_fp8_codes(got, want, pre_fn=None, what="fp8 codes") -> None:
    bad = fp8_mismatches(np.asarray(got), np.asarray(want))
    if bad.size == 0:
        return
    g0, w0 = np.asarray(got).reshape(-1)[bad[:5]], np.asarray(want).reshape(-1)[bad[:5]]
    assert pre_fn is not None and bad.size <= MAX_WINDOW_CASES, \
        f"{what}: {bad.size} mismatches, first {bad[:5]} got {g0} want {w0}"
    pre = pre_fn().reshape(-1)[bad]
    g = np.asarray(got).reshape(-1)[bad]
    w = np.asarray(want).reshape(-1)[bad]
    ok = near_mid(pre, E4_MIDS) & ((g & 0x80) == (w & 0x80))
    ok &= np.array([abs(E4_RANK.get(int(a) & 0x7F, -9) - E4_RANK.get(int(b) & 0x7F, 99)) == 1
                    for a, b in zip(g, w)], dtype=bool)
    assert ok.all(), f"{what}: {int((~ok).sum())} mismatches outside the midpoint window, " \
                     f"first {bad[~ok][:5]} got {g[~ok][:5]} want {w[~ok][:5]} pre {pre[~ok][:5]}"


def unpack_nibbles(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes).reshape(-1)
    out = np.empty(c.size * 2, dtype=np.uint8)
    out[0::2] = c & 0xF
    out[1::2] = c >> 4
    return out


def assert_fp4_codes(got, want, pre_fn=None, what="fp4 codes") -> None:
    g8 = np.asarray(got).reshape(-1)
    w8 = np.asarray(want).reshape(-1)
    if np.array_equal(g8, w8):
        return
    g = unpack_nibbles(g8)
    w = unpack_nibbles(w8)
    bad = np.flatnonzero(g != w)
    assert pre_fn is not None and bad.size <= MAX_WINDOW_CASES, \
        f"{what}: {bad.size} nibble mismatches, first {bad[:5]} got {g[bad[:5]]} want {w[bad[:5]]}"
    pre = pre_fn().reshape(-1)[bad]
    gb, wb = g[bad], w[bad]
    ok = near_mid(pre, E2_MIDS) & ((gb & 8) == (wb & 8))
    ok &= np.abs(np.array([E2_RANK[int(a) & 7] for a in gb]) - np.array([E2_RANK[int(b) & 7] for b in wb])) == 1
    assert ok.all(), f"{what}: {int((~ok).sum())} nibble mismatches outside the midpoint window, " \
                     f"first {bad[~ok][:5]} got {gb[~ok][:5]} want {wb[~ok][:5]} pre {pre[~ok][:5]}"
