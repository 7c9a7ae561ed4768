"""GPU: the library's E4M3/E2M1 conversions and its reciprocal-corrected
division against the oracle (through the C ABI entry point hq_convert and
the K128 quantizer)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from _compare import assert_fp8_codes

pytestmark = pytest.mark.gpu


def _bits_sweep(exp_lo: int, exp_hi: int, stride: int) -> np.ndarray:
    """Every `stride`-th binary32 pattern with unbiased exponent in [exp_lo, exp_hi], both signs,
    plus all patterns within 4 ulp of every multiple of 2^17 in the mantissa (E4M3/E2M1 midpoints)."""
    parts = []
    for e in range(exp_lo, exp_hi + 1):
        base = np.uint32((e + 127) << 23)
        mant = np.arange(0, 1 << 23, stride, dtype=np.uint32)
        parts.append(base | mant)
        grid = np.arange(0, 1 << 23, 1 << 17, dtype=np.int64)
        near = (grid[:, None] + np.arange(-4, 5)[None, :]).reshape(-1)
        near = near[(near >= 0) & (near < (1 << 23))].astype(np.uint32)
        parts.append(base | near)
    u = np.concatenate(parts)
    u = np.concatenate([u, u | np.uint32(0x80000000)])
    return u.view(np.float32)


def _gpu_convert(hq, fmt, x: np.ndarray) -> np.ndarray:
    xd = torch.from_numpy(x).cuda()
    out = torch.empty(x.size, dtype=torch.uint8, device="cuda")
    hq.hq_convert(fmt, xd, out, x.size)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def test_e4m3_conversion_matches_oracle(hq):
    x = _bits_sweep(-12, 9, 7)
    specials = np.array([0.0, -0.0, 448.0, 449.0, 464.0, 465.0, 1e30, -1e30, 2.0 ** -10, -(2.0 ** -10),
                         np.inf, -np.inf], dtype=np.float32)
    x = np.concatenate([x, specials])
    got = _gpu_convert(hq, hq.HQ_FMT_E4M3, x)
    want = oracle.encode_array(oracle.E4M3, x)
    assert_fp8_codes(got, want)
    # NaN stays NaN
    nan = _gpu_convert(hq, hq.HQ_FMT_E4M3, np.array([np.nan, -np.nan], dtype=np.float32))
    assert np.all((nan & 0x7F) == 0x7F)


def test_stochastic_e2m1_conversion_matches_oracle(hq):
    """The device's stochastic E2M1 routine (the one hq_group_rht_quant_sr
    uses) against the oracle's rule, element by element: a sweep of binary32
    patterns over and around the E2M1 range with seeded random bytes, every
    byte value for grid points, midpoints and values whose fraction is r/256
    exactly or just above it, both zeros, saturation and infinities, and a
    length that leaves a ragged group of four."""
    rng = np.random.default_rng(77)
    x = _bits_sweep(-8, 3, 17)
    r = rng.integers(0, 256, size=x.size, dtype=np.uint8)
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float32)
    steps = np.array([0.5, 0.5, 0.5, 0.5, 1.0, 1.0, 2.0], dtype=np.float32)
    special = [0.0, -0.0, 6.0, -6.0, 6.5, 7.0, 1e30, -1e30, np.inf, -np.inf, 5.999999, 1e-40, -1e-40]
    for g, st in zip(grid[:-1], steps):
        for f in (0, 1, 127, 128, 129, 254, 255):
            v = np.float32(g + st * f / 256.0)
            special += [v, -v, np.nextafter(v, np.float32(np.inf)), -np.nextafter(v, np.float32(np.inf))]
    sp = np.array(special, dtype=np.float32)
    xs = np.repeat(sp, 256)
    rs = np.tile(np.arange(256, dtype=np.uint8), sp.size)
    x = np.concatenate([x, xs, np.array([1.3, -2.6, 4.9], dtype=np.float32)])
    r = np.concatenate([r, rs, np.array([7, 200, 99], dtype=np.uint8)])
    assert x.size % 4 != 0
    xd, rd = torch.from_numpy(x).cuda(), torch.from_numpy(r).cuda()
    out = torch.empty(x.size, dtype=torch.uint8, device="cuda")
    hq.hq_convert_e2m1_sr(xd, rd, out, x.size)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    want = oracle.e2m1_sr(x, r).astype(np.uint8)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, (bad[:8], x[bad[:8]], r[bad[:8]], got[bad[:8]], want[bad[:8]])


def test_e2m1_conversion_matches_oracle(hq):
    x = _bits_sweep(-5, 4, 3)
    x = np.concatenate([x, np.array([0.0, -0.0, 6.0, 7.0, 1e30, -1e30, 5.0, -5.0], dtype=np.float32)])
    got = _gpu_convert(hq, hq.HQ_FMT_E2M1, x)
    want = oracle.encode_array(oracle.E2M1, x)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, (bad[:8], x[bad[:8]], got[bad[:8]], want[bad[:8]])


def test_reciprocal_corrected_division_is_ieee(hq):
    """The K128 quantizer's per-element division (RN(1/s) + two FMA remainder
    corrections) gives the same codes as the oracle's IEEE division on groups
    built to put y/s within a few ulp of E4M3 midpoints, and on wide random
    groups."""
    rng = np.random.default_rng(99)
    G = 20000
    amax = rng.uniform(2.0 ** -20, 2.0 ** 20, G).astype(np.float32)
    s = (np.maximum(amax, np.float32(1e-10)) * (np.float32(1) / np.float32(448))).astype(np.float32)
    mids = np.array([1.0625, 1.1875, 3.25, 7.5, 13.0, 26.0, 52.0, 104.0, 208.0, 432.0, 0.0009765625,
                     0.0029296875, 0.0166015625], dtype=np.float64)
    y = np.empty((G, 128), dtype=np.float32)
    y[:, 0] = amax
    m = mids[rng.integers(0, mids.size, (G, 127))]
    y[:, 1:] = (m * s[:, None].astype(np.float64)).astype(np.float32)
    jit = rng.integers(-3, 4, (G, 127)).astype(np.int32)
    y[:, 1:] = (y[:, 1:].view(np.int32) + jit).view(np.float32)
    y[:, 1:] *= np.where(rng.random((G, 127)) < 0.5, -1, 1).astype(np.float32)
    y[: G // 4, 1:] = (rng.standard_normal((G // 4, 127)) * amax[: G // 4, None]).astype(np.float32) / 4
    y[: G // 4, 1:] = np.clip(y[: G // 4, 1:], -amax[: G // 4, None], amax[: G // 4, None])
    yd = torch.from_numpy(y).cuda()
    codes, scales = hq.swiglu_fp8_k128(hq.HQ_ACT_NONE_F32, yd, 128)
    want_c, want_s, _ = oracle.swiglu_fp8_k128(oracle.NONE_F32, y, G, 128)
    np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint32), want_s.view(np.uint32))
    np.testing.assert_array_equal(codes.cpu().numpy(), want_c)   # bit-exact, no window needed
