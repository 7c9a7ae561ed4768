"""Pins for the oracle's scale formats for direct GEMM consumption.

UE8M0 FP8 scales (the use_ue8m0 option raised in the TensorRT-LLM PR #15158
review): checked against the FP8 rule of the onnxruntime PR #33644
description recomputed here in binary32, the power-of-two rounding derived
from the exponent with Python's exact frexp, and exact rational nearest-even
E4M3 codes.  The interleaved 128 x 4 NVFP4 block-scale tiles (the tcgen05
scale-factor layout discussed in DeepGEMM issue #320): the offset function
against an independent numpy construction of the tile permutation, hand
values, bijectivity, and the wiring of the layout flag into every NVFP4
output of the oracle.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synthetic as S
from _exact import e4m3_grid, nearest_code

E4C, E4V = e4m3_grid()
F = np.float32


def ue8m0_ref(s: np.float32) -> float:
    """Smallest power of two >= s, from the exact binary expansion of s."""
    m, e = math.frexp(float(s))  # s = m 2^e, m in [0.5, 1)
    return float(s) if m == 0.5 else math.ldexp(1.0, e)


def groups_with_range(seed: int, n_groups: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    g = rng.standard_normal((n_groups, 128)) * np.exp2(rng.integers(-40, 40, (n_groups, 1)))
    g[0] = 0.0                      # all zero: the 1e-10 floor
    g[1] = 0.0
    g[1, 7] = 448.0                 # amax 448: s = 1 exactly, already a power of two
    g[2] = 0.0
    g[2, 3] = -3.0 * 2.0 ** -20     # s not a power of two
    g[3, :] = 2.0 ** -135           # subnormal-scale values
    return g.astype(np.float32)


def check_ue8m0_group(y: np.ndarray, codes: np.ndarray, scale: float) -> None:
    amax = F(np.max(np.abs(y)))
    s = F(F(max(amax, F(1e-10))) * F(1.0 / 448.0))  # the printed FP8 rule in binary32
    want = ue8m0_ref(s)
    assert float(scale) == want, (float(s), float(scale), want)
    m, _ = math.frexp(want)
    assert m == 0.5                                  # a power of two
    assert want >= float(s) > want / 2
    bits = np.array([scale], dtype=np.float32).view(np.uint32)[0]
    assert bits & 0x7FFFFF == 0                      # the UE8M0 byte is the exponent field alone
    for v, c in zip(y, codes):
        q = Fraction(float(v)) / Fraction(want)      # exact: a power of two
        assert abs(q) <= 448 * (1 + Fraction(1, 2 ** 20))  # no value needs saturation
        exp = nearest_code(q, E4C, E4V, 0x80, np.signbit(v))
        assert int(c) == exp, (float(v), want, int(c), exp)


def test_ue8m0_k128_against_exact_codes():
    g = groups_with_range(301, 40)
    x = g.reshape(4, 10 * 128)
    codes, scales, _ = oracle.swiglu_fp8_k128(oracle.NONE_F32 | oracle.UE8M0, x, 4, 10 * 128)
    for r in range(4):
        for k in range(10):
            check_ue8m0_group(x[r, 128 * k:128 * k + 128], codes[r, 128 * k:128 * k + 128], scales[r, k])


def test_ue8m0_dsa_against_exact_codes_and_plain_rule():
    M, G = 6, 3
    pe = S.normal_bf16(311, (M, G, 64))
    nope = S.with_outliers_bf16(S.normal_bf16(312, (M, G, 64)), 313, p=0.05, factor=1e4)
    ld = 8
    c_ue, s_ue, _ = oracle.cat_rotate_fp8(pe, nope, M, G, 128, scale_layout=oracle.TRANSPOSED | oracle.UE8M0,
                                          scale_ld=ld)
    c_pl, s_pl, _ = oracle.cat_rotate_fp8(pe, nope, M, G, 128, scale_layout=oracle.TRANSPOSED, scale_ld=ld)
    for t in range(M):
        for g in range(G):
            su = s_ue[g, t]
            assert float(su) == ue8m0_ref(s_pl[g, t])
            # with a plain scale that is a power of two already the two paths agree
            if math.frexp(float(s_pl[g, t]))[0] == 0.5:
                assert np.array_equal(c_ue[t, 128 * g:128 * g + 128], c_pl[t, 128 * g:128 * g + 128])
    # rotated values straight from the unrotated path (hadamard 0): y is the concatenated input
    c0, s0, _ = oracle.cat_rotate_fp8(pe, nope, M, G, 0, scale_layout=oracle.UE8M0)
    v = np.concatenate([S.bf16_bits_to_f32(pe), S.bf16_bits_to_f32(nope)], axis=-1)
    for t in range(M):
        for g in range(G):
            check_ue8m0_group(v[t, g], c0[t, 128 * g:128 * g + 128], s0[t, g])


# ------------------------------------------------------------------ layout
def swizzle_numpy(plain: np.ndarray) -> np.ndarray:
    """The interleaved tiles built by reshaping: rows r = 128 tr + 32 rq + ri,
    columns c = 4 tc + cc; bytes ordered (tr, tc, ri, rq, cc)."""
    R, C = plain.shape
    t = plain.reshape(R // 128, 4, 32, C // 4, 4)          # (tr, rq, ri, tc, cc)
    return np.ascontiguousarray(t.transpose(0, 3, 2, 1, 4)).reshape(-1)


def test_swizzle_offsets_match_reshape_construction():
    for R, C in ((128, 4), (256, 8), (384, 28)):
        plain = np.arange(R * C, dtype=np.int64).reshape(R, C)
        want = swizzle_numpy(plain)
        got = np.empty(R * C, dtype=np.int64)
        for r in range(R):
            for c in range(C):
                got[oracle.sf_swizzled_offset(r, c, C)] = plain[r, c]
        assert np.array_equal(got, want), (R, C)


def test_swizzle_hand_values_and_bijection():
    assert oracle.sf_swizzled_offset(0, 0, 4) == 0
    assert oracle.sf_swizzled_offset(33, 2, 4) == 16 * 1 + 4 * 1 + 2
    assert oracle.sf_swizzled_offset(127, 3, 4) == 511
    assert oracle.sf_swizzled_offset(0, 4, 8) == 512           # second tile along the columns
    assert oracle.sf_swizzled_offset(128, 0, 8) == 1024        # first tile of the second row of tiles
    offs = {oracle.sf_swizzled_offset(r, c, 12) for r in range(256) for c in range(12)}
    assert offs == set(range(256 * 12))


@pytest.mark.parametrize("rot", [False, True])
def test_grouped_swizzled_is_the_plain_layout_permuted(rot):
    splits = [128, 0, 256]
    M, K = sum(splits), 256
    x = S.normal_bf16(321, (M, K))
    mask = S.sign_mask16(322)
    fl = oracle.ROWWISE | oracle.COLWISE | (oracle.ROW_RHT if rot else 0)
    plain = oracle.group_rht_quant(x, splits, mask, fl)
    swz = oracle.group_rht_quant(x, splits, mask, fl | oracle.SF_SWIZZLED)
    for k in ("row_codes", "col_codes", "amax_row", "amax_col", "sdec_row", "sdec_col"):
        assert np.array_equal(plain[k].view(np.uint8), swz[k].view(np.uint8)), k
    assert np.array_equal(swz["row_sf"].reshape(-1), swizzle_numpy(plain["row_sf"].reshape(M, K // 16)))
    r0 = 0
    for Ms in splits:
        if Ms:
            base = K * r0 // 16
            blk = plain["col_sf"][base:base + K * Ms // 16].reshape(K, Ms // 16)
            assert np.array_equal(swz["col_sf"][base:base + K * Ms // 16], swizzle_numpy(blk))
        r0 += Ms


def test_dsa_nvfp4_swizzled_block_scales():
    M, G = 128, 2
    pe = S.normal_bf16(331, (M, G, 64))
    nope = S.normal_bf16(332, (M, G, 64))
    plain = oracle.cat_rotate_nvfp4(pe, nope, M, G, 128)
    swz = oracle.cat_rotate_nvfp4(pe, nope, M, G, 128, scale_layout=oracle.ROWMAJOR | oracle.SF_SWIZZLED)
    assert np.array_equal(plain["codes"], swz["codes"]) and np.array_equal(plain["sdec"], swz["sdec"])
    assert np.array_equal(swz["block_sf"].reshape(-1), swizzle_numpy(plain["block_sf"]))
    with pytest.raises(ValueError):  # rows must fill whole tiles
        oracle.cat_rotate_nvfp4(pe[:64], nope[:64], 64, G, 128, scale_layout=oracle.SF_SWIZZLED)
