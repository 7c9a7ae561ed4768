"""Pins for the CPU oracle: each test ties it to something other than itself.

Sources: the format bit-field definitions (E4M3, E2M1), exact rational brute
force, scipy's Sylvester Hadamard matrix, torch's float8_e4m3fn cast, FP64
exp, closed forms and invariants the pages state (orthonormal rotation,
(Hq).(Hk) = q.k from the TensorRT-LLM PR #15158 discussion; the FP8 scale
rule of the onnxruntime PR #33644 description).
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
import synthetic as S
from _exact import e2m1_grid, e4m3_grid, frac, is_negative, near_midpoint, nearest_code

E4C, E4V = e4m3_grid()
E2C, E2V = e2m1_grid()
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32(bits: int) -> np.float32:
    return np.array([bits], dtype=np.uint32).view(np.float32)[0]


def _interesting_e4m3_values():
    vals = []
    for lo, hi in zip(E4V[:-1], E4V[1:]):
        mid = (lo + hi) / 2
        m = np.float32(float(mid))
        vals += [m, np.nextafter(m, np.float32(np.inf)), np.nextafter(m, np.float32(-np.inf)),
                 np.float32(float(lo)), np.float32(float(hi))]
    vals += [np.float32(v) for v in (0.0, 448.0, 449.0, 464.0, 464.0001, 480.0, 1e6, 3e38, 2.0 ** -9,
                                      2.0 ** -10, 2.0 ** -10 * 1.0001, 1e-30, 1e-45)]
    rng = np.random.default_rng(5)
    vals += list((rng.standard_normal(20000) * np.exp2(rng.integers(-14, 10, 20000))).astype(np.float32))
    arr = np.array(vals, dtype=np.float32)
    return np.concatenate([arr, -arr])


# ----------------------------------------------------------------- E4M3
def test_e4m3_decode_matches_bitfield_definition():
    for code, v in zip(E4C, E4V):
        assert oracle.e4m3_decode(code) == float(v)
        assert oracle.e4m3_decode(code | 0x80) == -float(v)
    assert math.isnan(oracle.e4m3_decode(0x7F)) and math.isnan(oracle.e4m3_decode(0xFF))
    assert oracle.e4m3_decode(0x7E) == 448.0


def test_e4m3_encode_is_nearest_even_saturating():
    """Brute force: nearest E4M3 value by exact distance, ties to the even code."""
    x = _interesting_e4m3_values()
    got = oracle.encode_array(oracle.E4M3, x)
    for v, c in zip(x, got):
        want = nearest_code(frac(v), E4C, E4V, 0x80, is_negative(v))
        assert c == want, (float(v), hex(c), hex(want))


def test_e4m3_encode_matches_torch_cast_in_range():
    """torch's float32 -> float8_e4m3fn cast (round to nearest even) agrees below 448."""
    rng = np.random.default_rng(11)
    x = (rng.standard_normal(200000) * np.exp2(rng.integers(-16, 9, 200000))).astype(np.float32)
    x = x[np.abs(x) < 448]
    x = np.concatenate([x, _interesting_e4m3_values()])
    x = x[np.abs(x) < 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.encode_array(oracle.E4M3, x)
    np.testing.assert_array_equal(got, ref)


def test_e4m3_special_values():
    assert oracle.e4m3_encode(float("inf")) == 0x7E
    assert oracle.e4m3_encode(float("-inf")) == 0xFE
    assert oracle.e4m3_encode(float("nan")) & 0x7F == 0x7F
    assert oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(-1e-30) == 0x80


# ----------------------------------------------------------------- E2M1
def test_e2m1_grid_and_decode():
    assert [float(v) for v in E2V] == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    for code, v in zip(E2C, E2V):
        assert oracle.e2m1_decode(code) == float(v)
        assert oracle.e2m1_decode(code | 8) == -float(v)


def test_e2m1_encode_is_nearest_even_saturating():
    vals = []
    for lo, hi in zip(E2V[:-1], E2V[1:]):
        m = np.float32(float((lo + hi) / 2))
        vals += [m, np.nextafter(m, np.float32(9)), np.nextafter(m, np.float32(-9)), np.float32(float(lo))]
    vals += [np.float32(v) for v in (6.0, 6.5, 7.0, 100.0, 1e30, 0.0, 1e-40)]
    rng = np.random.default_rng(3)
    vals += list((rng.standard_normal(20000) * 3).astype(np.float32))
    x = np.array(vals, dtype=np.float32)
    x = np.concatenate([x, -x])
    got = oracle.encode_array(oracle.E2M1, x)
    for v, c in zip(x, got):
        assert c == nearest_code(frac(v), E2C, E2V, 0x8, is_negative(v)), float(v)
    # the tie cases spelled out: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for v, want in ties.items():
        assert oracle.e2m1_decode(oracle.e2m1_encode(v)) == want


# ------------------------------------------------------------- Hadamard
@pytest.mark.parametrize("n", [2, 4, 16, 128])
def test_fwht_columns_equal_scipy_sylvester_matrix(n):
    """The butterfly on unit vectors reproduces scipy.linalg.hadamard exactly."""
    H = scipy.linalg.hadamard(n)
    for j in range(n):
        e = np.zeros(n, dtype=np.float32)
        e[j] = 1
        np.testing.assert_array_equal(oracle.fwht(e), H[:, j].astype(np.float32))
    assert np.array_equal(H @ H.T, n * np.eye(n, dtype=H.dtype))


def test_fwht_by_hand_n4():
    # H4 (Sylvester) * [1, 2, 3, 4] = [10, -2, -4, 0]
    np.testing.assert_array_equal(oracle.fwht(np.array([1, 2, 3, 4], np.float32)), [10, -2, -4, 0])


@pytest.mark.parametrize("n", [16, 128])
def test_fwht_matches_dense_fp64_within_norm_tolerance(n):
    rng = np.random.default_rng(n)
    H = scipy.linalg.hadamard(n).astype(np.float64)
    for _ in range(200):
        x = (rng.standard_normal(n) * np.exp2(rng.integers(-4, 5))).astype(np.float32)
        y = oracle.fwht(x).astype(np.float64) / math.sqrt(n)
        ref = H @ x.astype(np.float64) / math.sqrt(n)
        assert np.max(np.abs(y - ref)) <= 1e-5 * np.linalg.norm(x)
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) <= 1e-6 * np.linalg.norm(x)


def test_c128_is_nearest_binary32_to_two_pow_minus_3_5():
    c = frac(f32(0x3DB504F3))
    ulp = Fraction(2) ** (-4 - 23)   # c lies in [2^-4, 2^-3)
    lo, hi = c - ulp / 2, c + ulp / 2
    assert lo * lo < Fraction(1, 128) < hi * hi


# -------------------------------------------------------- FP8 1x128 rule
def _golden_rule():
    vals = {}
    for line in open(os.path.join(GOLDEN, "fp8_scale_rule.txt")):
        if line.strip() and not line.startswith("#"):
            k, v = line.split()
            vals[k] = float(v)
    return vals


def _check_fp8_groups(y32, codes, scales):
    """Codes are the exact nearest E4M3 of y/s (allowed to differ only inside
    the 2^-20 midpoint window); scales follow the page's rule."""
    rule = _golden_rule()
    floor = np.float32(rule["amax_floor"])
    inv = np.float32(1) / np.float32(rule["divisor"])
    assert inv.view(np.uint32) == 0x3B124925 and floor.view(np.uint32) == 0x2EDBE6FF
    G = int(rule["group_size"])
    y = y32.reshape(-1, G)
    codes = codes.reshape(-1, G)
    scales = scales.reshape(-1)
    for g in range(y.shape[0]):
        amax = np.max(np.abs(y[g]))
        s = np.float32(max(amax, floor)) * inv
        assert scales[g] == s
        for v, c in zip(y[g], codes[g]):
            q = frac(v) / frac(s)
            want = nearest_code(q, E4C, E4V, 0x80, is_negative(v))
            if c != want:
                assert near_midpoint(q, E4V), (float(v), hex(c), hex(want))
        if amax > floor:
            k = int(np.argmax(np.abs(y[g])))
            assert codes[g][k] & 0x7F == 0x7E   # the amax element lands on 448


def test_fp8_1x128_no_rotation_brute_force():
    rng = np.random.default_rng(7)
    M = 24
    x = S.f32_to_bf16_bits((rng.standard_normal((M, 128)) * np.exp2(rng.integers(-8, 8, (M, 1)))).astype(np.float32))
    x[3] = 0                               # zero group: scale = 1e-10/448, codes 0
    codes, scales, _ = oracle.cat_rotate_fp8(x, None, M, 1, hadamard_n=0)
    _check_fp8_groups(S.bf16_bits_to_f32(x), codes, scales)
    assert np.all(codes[3] == 0)


def test_fp8_rotation_is_orthonormal_hadamard_of_concat():
    """cat(pe, nope) -> H128/sqrt(128) -> quant: dequantized values match the
    dense FP64 rotation within the FP8 bound, the rotation preserves the norm,
    and (Hq).(Hk) = q.k holds for the rotated FP32 values."""
    rng = np.random.default_rng(8)
    M, G = 16, 3
    pe = S.normal_bf16(21, (M, G, 64))
    nope = S.normal_bf16(22, (M, G, 64))
    codes, scales, pre = oracle.cat_rotate_fp8(pe, nope, M, G, hadamard_n=128, want_pre=True)
    H = scipy.linalg.hadamard(128).astype(np.float64) / math.sqrt(128)
    v = np.concatenate([S.bf16_bits_to_f32(pe), S.bf16_bits_to_f32(nope)], axis=-1).astype(np.float64)
    y_ref = v @ H.T                                      # [M, G, 128]
    y = pre.reshape(M, G, 128).astype(np.float64) * scales.reshape(M, G, 1)
    norms = np.linalg.norm(v, axis=-1, keepdims=True)
    assert np.max(np.abs(y - y_ref) / norms) <= 1e-5    # rotated FP32 within 1e-5 of row norm
    # (Hq).(Hk) = q.k on the rotated values
    assert np.allclose(np.einsum("mgi,mgi->mg", y[:, :1], y[:, 1:2]),
                       np.einsum("mgi,mgi->mg", v[:, :1], v[:, 1:2]), rtol=1e-4, atol=1e-4)
    deq = np.array([oracle.e4m3_decode(c) for c in codes.reshape(-1)]).reshape(M, G, 128) * scales.reshape(M, G, 1)
    # E4M3 relative step is 2^-3: error <= half a step of the value's binade,
    # or half the subnormal step 2^-10 * s near zero
    bound = np.maximum(np.abs(y_ref) * 2.0 ** -4, scales.reshape(M, G, 1) * 2.0 ** -10) * 1.001
    assert np.all(np.abs(deq - y_ref) <= bound + 1e-6 * norms)
    # rotation matters: without it the codes differ
    codes0, _, _ = oracle.cat_rotate_fp8(pe, nope, M, G, hadamard_n=0)
    assert np.mean(codes0 != codes) > 0.5


def test_fp8_concat_order_and_transposed_scale_layout():
    M, G = 8, 5
    pe = S.normal_bf16(31, (M, G, 64))
    nope = S.normal_bf16(32, (M, G, 64))
    c_rm, s_rm, _ = oracle.cat_rotate_fp8(pe, nope, M, G, hadamard_n=0)
    c_tr, s_tr, _ = oracle.cat_rotate_fp8(pe, nope, M, G, hadamard_n=0, scale_layout=oracle.TRANSPOSED, scale_ld=12)
    np.testing.assert_array_equal(c_rm, c_tr)
    for t in range(M):
        for g in range(G):
            assert s_tr[g, t] == s_rm[t, g]
    # pe first: group (t, g) without rotation equals the plain quant of cat(pe, nope)
    flat = np.concatenate([pe, nope], axis=-1).reshape(M * G, 128)
    c_flat, s_flat, _ = oracle.cat_rotate_fp8(flat, None, M * G, 1, hadamard_n=0)
    np.testing.assert_array_equal(c_flat.reshape(M, G * 128), c_rm)
    np.testing.assert_array_equal(s_flat.reshape(M, G), s_rm)


def test_fp8_nan_stays_nan_and_inf_group():
    x = S.normal_bf16(41, (2, 128))
    x[0, 5] = 0x7FC0                      # NaN
    x[1, 9] = 0x7F80                      # +inf
    codes, scales, _ = oracle.cat_rotate_fp8(x, None, 2, 1, hadamard_n=0)
    assert codes[0, 5] & 0x7F == 0x7F     # NaN element stays NaN
    assert np.all((codes[0, np.arange(128) != 5] & 0x7F) != 0x7F)   # the rest stay finite
    assert np.isfinite(scales[0, 0])
    assert np.isinf(scales[1, 0]) and codes[1, 9] & 0x7F == 0x7F


# ------------------------------------------------------------ SwiGLU exp
def test_exp_within_two_ulp_of_fp64():
    x = np.concatenate([
        np.linspace(-103.9, 88.7, 400001, dtype=np.float32),
        (np.random.default_rng(2).standard_normal(200000) * 4).astype(np.float32),
        np.float32([0.0, -0.0, 1e-30, -1e-30, 88.72, -87.3, -100.0]),
    ])
    got = oracle.exp_f32(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    tiny = np.float64(2.0 ** -149)
    ulp = np.maximum(np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64), tiny)
    err = np.abs(got - ref) / ulp
    assert np.max(err) <= 2.0, float(np.max(err))
    assert oracle.exp_f32(np.float32([100.0]))[0] == np.inf
    assert oracle.exp_f32(np.float32([-200.0]))[0] == 0.0
    assert np.isnan(oracle.exp_f32(np.float32([np.nan]))[0])


def test_fp8_amax_outputs():
    """amax_opt: max |y| of each group (exact max |x| without rotation; the
    dense FP64 rotation's maximum within FP32 rounding with it), stored in the
    scales' layout, with s = max(amax, 1e-10) * RN(1/448) in binary32."""
    M, G = 12, 3
    xa = S.normal_bf16(301, (M, G, 64))
    xb = S.normal_bf16(302, (M, G, 64))
    xa[5, 1] = 0
    xb[5, 1] = 0                                   # an all-zero group
    inv = np.float32(1) / np.float32(448)
    _, sc, _, am = oracle.cat_rotate_fp8(xa, xb, M, G, 0, want_amax=True)
    v = np.concatenate([S.bf16_bits_to_f32(xa), S.bf16_bits_to_f32(xb)], axis=-1)
    np.testing.assert_array_equal(am, np.max(np.abs(v), axis=-1))
    np.testing.assert_array_equal(sc, np.maximum(am, np.float32(1e-10)) * inv)
    assert am[5, 1] == 0
    _, sct, _, amt = oracle.cat_rotate_fp8(xa, xb, M, G, 128, scale_layout=oracle.TRANSPOSED,
                                           scale_ld=16, want_amax=True)
    H = scipy.linalg.hadamard(128).astype(np.float64) / math.sqrt(128)
    ref = np.max(np.abs(v.astype(np.float64) @ H.T), axis=-1)      # [M, G]
    assert amt.shape == (G, 16)
    np.testing.assert_allclose(amt[:, :M].T, ref, rtol=2e-6)
    assert np.all(amt[:, M:] == 0)
    np.testing.assert_array_equal(sct[:, :M], np.maximum(amt[:, :M], np.float32(1e-10)) * inv)
    x = S.normal_f32(303, (4, 512))
    _, s1, _, a1 = oracle.swiglu_fp8_k128(oracle.NONE_F32, x, 4, 512, want_amax=True)
    np.testing.assert_array_equal(a1, np.max(np.abs(x.reshape(4, 4, 128)), axis=-1))
    np.testing.assert_array_equal(s1, np.maximum(a1, np.float32(1e-10)) * inv)


def test_swiglu_k128_values_and_rule():
    M, K = 6, 256
    gu = S.normal_f32(51, (M, 2 * K), std=math.sqrt(2.0))
    codes, scales, pre = oracle.swiglu_fp8_k128(oracle.SWIGLU_F32, gu, M, K, want_pre=True)
    g = gu[:, :K].astype(np.float64)
    u = gu[:, K:].astype(np.float64)
    act_ref = g / (1.0 + np.exp(-g)) * u
    act = pre.astype(np.float64) * np.repeat(scales, 128, axis=1)
    assert np.max(np.abs(act - act_ref) / (np.abs(act_ref) + 1e-30)) < 2e-6
    # the K128 rule on the FP32 activations: rebuild them (they are pre * s up
    # to one rounding) from FP64, round once to FP32, and brute-force the codes
    act32 = act_ref.astype(np.float32)
    c2, s2, _ = oracle.swiglu_fp8_k128(oracle.NONE_F32, act32, M, K)
    _check_fp8_groups(act32, c2, s2)


def test_k128_bf16_equals_f32_of_same_values():
    x = S.normal_bf16(61, (4, 384))
    a, sa, _ = oracle.swiglu_fp8_k128(oracle.NONE_BF16, x, 4, 384)
    b, sb, _ = oracle.swiglu_fp8_k128(oracle.NONE_F32, S.bf16_bits_to_f32(x), 4, 384)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(sa, sb)
    _check_fp8_groups(S.bf16_bits_to_f32(x), a, sa)


# ----------------------------------------------------------------- NVFP4
def _unpack(codes):
    lo = codes & 0xF
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(*codes.shape[:-1], codes.shape[-1] * 2)


def _e2m1_vals(nibbles):
    return np.array([oracle.e2m1_decode(int(c)) for c in nibbles.reshape(-1)]).reshape(nibbles.shape)


def _e4m3_vals(codes):
    return np.array([oracle.e4m3_decode(int(c)) for c in codes.reshape(-1)]).reshape(codes.shape)


def _rht_dense(x_blocks, mask):
    """0.25 * H16 * diag(sigma) applied to the last axis (FP64, scipy's H)."""
    H = scipy.linalg.hadamard(16).astype(np.float64)
    sigma = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(16)])
    return 0.25 * (x_blocks * sigma) @ H.T


def _nvfp4_case(seed=71, K=256, splits=(128, 0, 256, 128), mask=0xA5C3):
    M = sum(splits)
    x = S.normal_bf16(seed, (M, K))
    # give sections very different magnitudes
    xf = S.bf16_bits_to_f32(x).copy()
    r0 = 0
    for i, m in enumerate(splits):
        xf[r0:r0 + m] *= np.float32(4.0 ** (i - 1))
        r0 += m
    x = S.f32_to_bf16_bits(xf)
    x = S.with_outliers_bf16(x, seed + 1, p=0.002)
    return x, list(splits), mask


def test_nvfp4_rowwise_codes_scales_and_global():
    x, splits, mask = _nvfp4_case()
    r = oracle.group_rht_quant(x, splits, mask, oracle.ROWWISE | oracle.COLWISE, want_pre=True)
    xf = S.bf16_bits_to_f32(x)
    M, K = x.shape
    r0 = 0
    for s, Ms in enumerate(splits):
        sec = xf[r0:r0 + Ms]
        A = np.float32(np.max(np.abs(sec))) if Ms else np.float32(0)
        assert r["amax_row"][s] == A
        S_enc = np.float32(2688) / A if A > 0 else np.float32(1)
        assert r["sdec_row"][s] == np.float32(1) / S_enc
        if Ms == 0:
            assert r["sdec_row"][s] == 1 and r["sdec_col"][s] == 1 and r["amax_col"][s] == 0
            continue
        blocks = sec.reshape(Ms, K // 16, 16)
        ab = np.max(np.abs(blocks), axis=-1)
        sf = r["row_sf"][r0:r0 + Ms]
        # block scale: nearest E4M3 of (a_b / 6) * S_enc (exact rational, window allowed)
        for i in range(0, Ms, 37):
            for kb in range(K // 16):
                t = frac(ab[i, kb]) / 6 * frac(S_enc)
                want = nearest_code(t, E4C, E4V, 0x80, False)
                if sf[i, kb] != want:
                    assert near_midpoint(t, E4V)
        # the block holding the section amax gets scale 448
        i, kb = np.unravel_index(np.argmax(ab), ab.shape)
        assert sf[i, kb] == 0x7E
        # codes: nearest E2M1 of the pre-rounding value; element 2k in the low nibble
        nib = _unpack(r["row_codes"][r0:r0 + Ms])
        pre = r["row_pre"][r0:r0 + Ms]
        for (i, k) in zip(*np.nonzero(np.ones((Ms, K), bool)[::5])):
            i *= 5
            want = nearest_code(frac(pre[i, k]), E2C, E2V, 0x8, is_negative(pre[i, k]))
            if nib[i, k] != want:
                assert near_midpoint(frac(pre[i, k]), E2V)
        # pre = x * enc with enc = S_enc / sf
        sff = _e4m3_vals(sf)
        enc = np.where(sff == 0, 0, np.float32(S_enc) / sff.astype(np.float32)).astype(np.float32)
        np.testing.assert_array_equal(pre, (blocks * enc[..., None]).reshape(Ms, K).astype(np.float32))
        # dequantized rows reconstruct x within the NVFP4 bound
        deq = _e2m1_vals(nib).reshape(Ms, K // 16, 16) * sff[..., None] / np.float64(S_enc)
        assert np.all(np.abs(deq - blocks) <= ab[..., None] / 6 * 1.07 + 1e-30)
        r0 += Ms


def test_nvfp4_columnwise_is_transposed_rht_of_section():
    x, splits, mask = _nvfp4_case(seed=81)
    r = oracle.group_rht_quant(x, splits, mask, oracle.ROWWISE | oracle.COLWISE, want_pre=True)
    xf = S.bf16_bits_to_f32(x).astype(np.float64)
    M, K = x.shape
    r0 = 0
    for s, Ms in enumerate(splits):
        if Ms == 0:
            continue
        sec = xf[r0:r0 + Ms]                              # [Ms, K]
        blocks = sec.T.reshape(K, Ms // 16, 16)           # column c, 16-row block
        v_ref = _rht_dense(blocks, mask)                  # FP64, sigma on the input side
        A = r["amax_col"][s]
        assert abs(A - np.max(np.abs(v_ref))) <= 1e-6 * A
        S_enc = np.float32(2688) / A
        assert r["sdec_col"][s] == np.float32(1) / S_enc
        cc = r["col_codes"][K * r0 // 2: K * (r0 + Ms) // 2].reshape(K, Ms // 2)
        cs = r["col_sf"][K * r0 // 16: K * (r0 + Ms) // 16].reshape(K, Ms // 16)
        pre = r["col_pre"][K * r0: K * (r0 + Ms)].reshape(K, Ms // 16, 16)
        sff = _e4m3_vals(cs)
        enc = np.where(sff == 0, 0, np.float64(S_enc) / sff)
        v = pre / np.where(enc == 0, 1, enc)[..., None]
        norms = np.linalg.norm(blocks, axis=-1, keepdims=True)
        assert np.max(np.abs(v - v_ref) / np.maximum(norms, 1e-30)) <= 1e-5
        # the inverse rotation of the dequantized columns gives back x (orthonormal)
        deq = _e2m1_vals(_unpack(cc)).reshape(K, Ms // 16, 16) * sff[..., None] / np.float64(S_enc)
        H = scipy.linalg.hadamard(16).astype(np.float64)
        sigma = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(16)])
        back = (0.25 * deq @ H) * sigma                   # (0.25 H D)^-1 = 0.25 D H^T, H symmetric
        err = np.linalg.norm(back - blocks, axis=-1)
        ab = np.max(np.abs(v_ref), axis=-1)
        assert np.all(err <= 4 * ab / 6 * 1.07 + 1e-30)
        r0 += Ms


def test_nvfp4_sign_mask_all_plus_reduces_to_plain_hadamard():
    x = S.normal_bf16(91, (128, 128))
    r = oracle.group_rht_quant(x, [128], 0x0000, oracle.COLWISE, want_pre=True)
    r2 = oracle.group_rht_quant(x, [128], 0xFFFF, oracle.COLWISE, want_pre=True)
    # sigma = -1 everywhere negates every rotated value: codes flip sign bits
    np.testing.assert_array_equal(r["col_sf"], r2["col_sf"])
    n1, n2 = _unpack(r["col_codes"]).reshape(-1), _unpack(r2["col_codes"]).reshape(-1)
    nz = r["col_pre"] != 0
    np.testing.assert_array_equal(n1[nz] ^ 8, n2[nz])
    np.testing.assert_array_equal(r["col_pre"][nz], -r2["col_pre"][nz])
    # and with sigma = +1 the rotation is the scipy Sylvester matrix / 4
    blocks = S.bf16_bits_to_f32(x).astype(np.float64).T.reshape(128, 8, 16)
    H = scipy.linalg.hadamard(16).astype(np.float64)
    sff = _e4m3_vals(r["col_sf"].reshape(128, 8))
    S_enc = np.float32(2688) / r["amax_col"][0]
    v = r["col_pre"].reshape(128, 8, 16) / (np.float64(S_enc) / sff)[..., None]
    assert np.max(np.abs(v - 0.25 * blocks @ H.T)) <= 1e-5 * np.max(np.linalg.norm(blocks, axis=-1))


def test_nvfp4_flags_select_directions_and_reject_bad_splits():
    x = S.normal_bf16(95, (256, 128))
    both = oracle.group_rht_quant(x, [128, 128], 0x1234, oracle.ROWWISE | oracle.COLWISE)
    row = oracle.group_rht_quant(x, [128, 128], 0x1234, oracle.ROWWISE)
    col = oracle.group_rht_quant(x, [128, 128], 0x1234, oracle.COLWISE)
    for k in ("row_codes", "row_sf", "amax_row", "sdec_row"):
        np.testing.assert_array_equal(both[k], row[k])
    for k in ("col_codes", "col_sf", "amax_col", "sdec_col"):
        np.testing.assert_array_equal(both[k], col[k])
    with pytest.raises(ValueError):
        oracle.group_rht_quant(x, [64, 192], 0, oracle.ROWWISE)       # not a multiple of 128
    with pytest.raises(ValueError):
        oracle.group_rht_quant(x, [128], 0, oracle.ROWWISE)           # splits do not sum to M


def test_nvfp4_row_rht_is_rotation_along_k():
    """ROW_RHT: every 16-element row block is rotated (sigma by position in the
    block) before the rowwise amax and cast; checked against a dense FP64
    rotation, the inverse rotation of the dequantized rows and the plain cast
    when the flag is off."""
    x, splits, mask = _nvfp4_case(seed=83, splits=(256, 128, 0))
    r = oracle.group_rht_quant(x, splits, mask, oracle.ROWWISE | oracle.ROW_RHT, want_pre=True)
    plain = oracle.group_rht_quant(x, splits, mask, oracle.ROWWISE)
    assert not np.array_equal(r["row_codes"], plain["row_codes"])
    xf = S.bf16_bits_to_f32(x).astype(np.float64)
    M, K = x.shape
    H = scipy.linalg.hadamard(16).astype(np.float64)
    sigma = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(16)])
    r0 = 0
    for s, Ms in enumerate(splits):
        if Ms == 0:
            assert r["amax_row"][s] == 0 and r["sdec_row"][s] == 1
            continue
        blocks = xf[r0:r0 + Ms].reshape(Ms, K // 16, 16)
        v_ref = _rht_dense(blocks, mask)
        A = r["amax_row"][s]
        assert abs(A - np.max(np.abs(v_ref))) <= 1e-6 * A
        S_enc = np.float32(2688) / A
        assert r["sdec_row"][s] == np.float32(1) / S_enc
        sf = r["row_sf"][r0:r0 + Ms]
        sff = _e4m3_vals(sf)
        enc = np.where(sff == 0, 0, np.float64(S_enc) / sff)
        pre = r["row_pre"][r0:r0 + Ms].reshape(Ms, K // 16, 16)
        v = pre / np.where(enc == 0, 1, enc)[..., None]
        norms = np.linalg.norm(blocks, axis=-1, keepdims=True)
        assert np.max(np.abs(v - v_ref) / np.maximum(norms, 1e-30)) <= 1e-5
        # block scales follow the rotated block maxima
        ab = np.max(np.abs(v_ref), axis=-1)
        i, kb = np.unravel_index(np.argmax(ab), ab.shape)
        assert sf[i, kb] == 0x7E
        nib = _unpack(r["row_codes"][r0:r0 + Ms]).reshape(Ms, K // 16, 16)
        deq = _e2m1_vals(nib) * sff[..., None] / np.float64(S_enc)
        back = (0.25 * deq @ H) * sigma
        err = np.linalg.norm(back - blocks, axis=-1)
        assert np.all(err <= 4 * ab / 6 * 1.07 + 1e-30)
        r0 += Ms


def test_nvfp4_row_rht_equals_column_rht_of_transpose():
    """Rotating rows along K of x is the columnwise transform of x^T (one
    section each way), whose transposed output is laid out like x's rows."""
    x = S.normal_bf16(85, (128, 256))
    mask = 0x5A3C
    r = oracle.group_rht_quant(x, [128], mask, oracle.ROWWISE | oracle.ROW_RHT)
    xt = np.ascontiguousarray(x.T)
    c = oracle.group_rht_quant(xt, [256], mask, oracle.COLWISE)
    np.testing.assert_array_equal(r["row_codes"].reshape(-1), c["col_codes"])
    np.testing.assert_array_equal(r["row_sf"].reshape(-1), c["col_sf"])
    assert r["amax_row"][0] == c["amax_col"][0] and r["sdec_row"][0] == c["sdec_col"][0]


def test_nvfp4_amax_given_single_pass():
    """AMAX_GIVEN: the section amax values are inputs.  Given the computed
    ones, every output equals the two-pass result; given others, the block
    scales and codes follow the closed-form rule from S_enc = 2688 / A_given
    (saturating when A_given is below the data's amax), and an empty section
    keeps its given amax with sdec = 1 / S_enc."""
    x, splits, mask = _nvfp4_case(seed=87, splits=(128, 0, 256))
    both = oracle.ROWWISE | oracle.COLWISE
    ref = oracle.group_rht_quant(x, splits, mask, both)
    same = oracle.group_rht_quant(x, splits, mask, both | oracle.AMAX_GIVEN,
                                  amax_row=ref["amax_row"], amax_col=ref["amax_col"])
    for k in ref:
        np.testing.assert_array_equal(same[k], ref[k], err_msg=k)
    rot = oracle.group_rht_quant(x, splits, mask, oracle.ROWWISE | oracle.ROW_RHT)
    rot2 = oracle.group_rht_quant(x, splits, mask, oracle.ROWWISE | oracle.ROW_RHT | oracle.AMAX_GIVEN,
                                  amax_row=rot["amax_row"])
    for k in rot:
        np.testing.assert_array_equal(rot2[k], rot[k], err_msg=k)

    given = np.array([2.0, 3.0, 0.25], dtype=np.float32) * np.maximum(ref["amax_row"], 1)
    r = oracle.group_rht_quant(x, splits, mask, oracle.ROWWISE | oracle.AMAX_GIVEN, want_pre=True,
                               amax_row=given)
    np.testing.assert_array_equal(r["amax_row"], given)
    S_encs = [np.float32(2688) / g for g in given]
    assert r["sdec_row"][1] == np.float32(1) / S_encs[1]          # empty section
    xf = S.bf16_bits_to_f32(x)
    M, K = x.shape
    r0 = 0
    for s, Ms in enumerate(splits):
        if Ms == 0:
            continue
        blocks = xf[r0:r0 + Ms].reshape(Ms, K // 16, 16)
        ab = np.max(np.abs(blocks), axis=-1)
        sf = r["row_sf"][r0:r0 + Ms]
        for i in range(0, Ms, 29):
            for kb in range(K // 16):
                t = frac(ab[i, kb]) / 6 * frac(S_encs[s])
                want = nearest_code(t, E4C, E4V, 0x80, False)
                if sf[i, kb] != want:
                    assert near_midpoint(t, E4V)
        sff = _e4m3_vals(sf)
        enc = np.where(sff == 0, 0, S_encs[s] / sff.astype(np.float32)).astype(np.float32)
        pre = r["row_pre"][r0:r0 + Ms]
        np.testing.assert_array_equal(pre, (blocks * enc[..., None]).reshape(Ms, K).astype(np.float32))
        nib = _unpack(r["row_codes"][r0:r0 + Ms])
        if given[s] < ref["amax_row"][s]:
            # below the data's amax: the top block scale saturates at 448 and
            # codes saturate at 6
            i, kb = np.unravel_index(np.argmax(ab), ab.shape)
            assert sf[i, kb] == 0x7E
            assert np.any((nib & 7) == 7)
        r0 += Ms
    # a given amax that is not positive (negative, NaN) acts like 0: S_enc = 1
    z = oracle.group_rht_quant(x, splits, mask, both | oracle.AMAX_GIVEN, amax_row=np.zeros(3, np.float32),
                               amax_col=np.zeros(3, np.float32))
    assert np.all(z["sdec_row"] == 1) and np.all(z["sdec_col"] == 1)
    bad = np.array([-1.0, np.nan, -0.0], dtype=np.float32)
    w = oracle.group_rht_quant(x, splits, mask, both | oracle.AMAX_GIVEN, amax_row=bad, amax_col=bad[::-1])
    for k in ("row_codes", "row_sf", "col_codes", "col_sf", "sdec_row", "sdec_col"):
        np.testing.assert_array_equal(w[k], z[k], err_msg=k)


def test_fp4_dsa_without_rotation_follows_the_nvfp4_rule():
    """cat -> NVFP4 per 128-vector (no rotation): vector amax, decode scale,
    block scales and codes follow the closed-form two-level rule."""
    M, G = 5, 3
    pe = S.normal_bf16(311, (M, G, 64))
    nope = S.with_outliers_bf16(S.normal_bf16(312, (M, G, 64)), 313, p=0.02)
    pe[2, 1] = 0
    nope[2, 1] = 0                                    # an all-zero vector
    r = oracle.cat_rotate_nvfp4(pe, nope, M, G, 0, want_pre=True, want_amax=True)
    v = np.concatenate([S.bf16_bits_to_f32(pe), S.bf16_bits_to_f32(nope)], axis=-1)   # [M, G, 128]
    A = np.max(np.abs(v), axis=-1)
    np.testing.assert_array_equal(r["amax"], A)
    nib = _unpack(r["codes"]).reshape(M, G, 8, 16)
    sf = r["block_sf"].reshape(M, G, 8)
    pre = r["pre"].reshape(M, G, 8, 16)
    for t in range(M):
        for g in range(G):
            if A[t, g] == 0:
                assert r["sdec"][t, g] == 1 and np.all(sf[t, g] == 0) and np.all((nib[t, g] & 7) == 0)
                continue
            S_enc = np.float32(2688) / A[t, g]
            assert r["sdec"][t, g] == np.float32(1) / S_enc
            blocks = v[t, g].reshape(8, 16)
            ab = np.max(np.abs(blocks), axis=-1)
            for k in range(8):
                want = nearest_code(frac(ab[k]) / 6 * frac(S_enc), E4C, E4V, 0x80, False)
                if sf[t, g, k] != want:
                    assert near_midpoint(frac(ab[k]) / 6 * frac(S_enc), E4V)
            assert sf[t, g, int(np.argmax(ab))] == 0x7E        # the block holding the amax
            sff = _e4m3_vals(sf[t, g]).astype(np.float32)
            enc = np.where(sff == 0, 0, S_enc / sff).astype(np.float32)
            np.testing.assert_array_equal(pre[t, g], (blocks * enc[:, None]).astype(np.float32))
            for k in range(8):
                for i in range(16):
                    want = nearest_code(frac(pre[t, g, k, i]), E2C, E2V, 0x8, is_negative(pre[t, g, k, i]))
                    if nib[t, g, k, i] != want:
                        assert near_midpoint(frac(pre[t, g, k, i]), E2V)


def test_fp4_dsa_rotation_and_layouts():
    """With the rotation: the pre-rounding values are the dense FP64 rotation
    times the block encode factors, the dequantized vector rotates back to
    x within the NVFP4 bound, the amax equals the FP8 path's, and the
    transposed layout puts vector (t, g) at sdec[g, t]."""
    M, G = 6, 4
    pe = S.normal_bf16(321, (M, G, 64))
    nope = S.normal_bf16(322, (M, G, 64))
    r = oracle.cat_rotate_nvfp4(pe, nope, M, G, 128, want_pre=True, want_amax=True)
    x = np.concatenate([S.bf16_bits_to_f32(pe), S.bf16_bits_to_f32(nope)], axis=-1).astype(np.float64)
    H = scipy.linalg.hadamard(128).astype(np.float64) / math.sqrt(128)
    y = x @ H.T                                                             # [M, G, 128]
    assert np.max(np.abs(r["amax"] - np.max(np.abs(y), axis=-1)) / r["amax"]) <= 2e-6
    _, _, _, am8 = oracle.cat_rotate_fp8(pe, nope, M, G, 128, want_amax=True)
    np.testing.assert_array_equal(r["amax"], am8)
    sff = _e4m3_vals(r["block_sf"]).reshape(M, G, 8)
    S_enc = (1.0 / r["sdec"].astype(np.float64))[..., None]
    enc = np.where(sff == 0, 0, S_enc / sff)
    v = r["pre"].reshape(M, G, 8, 16) / np.where(enc == 0, 1, enc)[..., None]
    assert np.max(np.abs(v.reshape(M, G, 128) - y)) <= 1e-5 * np.max(np.linalg.norm(x, axis=-1))
    deq = _e2m1_vals(_unpack(r["codes"])).reshape(M, G, 8, 16) * (sff / S_enc)[..., None]
    back = deq.reshape(M, G, 128) @ H                                       # H orthonormal, symmetric
    ab = np.max(np.abs(y.reshape(M, G, 8, 16)), axis=-1)
    err = np.linalg.norm(back - x, axis=-1)
    assert np.all(err <= np.linalg.norm(ab / 6 * 1.07, axis=-1) * 4 + 1e-30)
    rt = oracle.cat_rotate_nvfp4(pe, nope, M, G, 128, scale_layout=oracle.TRANSPOSED, scale_ld=8)
    np.testing.assert_array_equal(rt["sdec"][:, :M], r["sdec"].T)
    assert np.all(rt["sdec"][:, M:] == 0)
    np.testing.assert_array_equal(rt["codes"], r["codes"])


# ------------------------------------------------ stochastic rounding
def _curand_words(seed, offset, n):
    """cuRAND's host-side Philox4x32-10 generator (a library routine on the
    CPU): n uint32 outputs of `seed` from output number `offset`."""
    import ctypes
    path = "/usr/local/cuda/lib64/libcurand.so"
    if not os.path.exists(path):
        pytest.skip("libcurand not present")
    L = ctypes.CDLL(path)
    L.curandSetPseudoRandomGeneratorSeed.argtypes = [ctypes.c_void_p, ctypes.c_ulonglong]
    L.curandSetGeneratorOffset.argtypes = [ctypes.c_void_p, ctypes.c_ulonglong]
    L.curandGenerate.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t]
    g = ctypes.c_void_p()
    assert L.curandCreateGeneratorHost(ctypes.byref(g), 161) == 0       # CURAND_RNG_PSEUDO_PHILOX4_32_10
    assert L.curandSetPseudoRandomGeneratorSeed(g, seed) == 0
    assert L.curandSetGeneratorOffset(g, offset) == 0
    out = np.zeros(n, dtype=np.uint32)
    assert L.curandGenerate(g, out.ctypes.data, n) == 0
    L.curandDestroyGenerator(g)
    return out


@pytest.mark.parametrize("seed", [0, 1, 0x0123456789ABCDEF, 2**64 - 1])
def test_philox_matches_curand_host_generator(seed):
    """The oracle's Philox4x32-10 against cuRAND's host generator (a library
    routine on the CPU).  Its output block i is Philox with counter
    (i >> 16, 0, i & 0xFFFF, 0) and key = the seed's halves (observed layout
    of its default ordering), which exercises counter words 0 and 2 and the
    key; words 1 and 3 enter only through the same XORs as the key."""
    for i in (0, 1, 65535, 65536, 65536 * 7 + 123, (1 << 47) + 5):
        w = _curand_words(seed, 4 * i, 4)
        got = oracle.philox4x32_10([i >> 16 & 0xFFFFFFFF, 0, i & 0xFFFF, 0], [seed & 0xFFFFFFFF, seed >> 32])
        np.testing.assert_array_equal(got, w, err_msg=f"block {i}")


def test_e2m1_stochastic_rounding_rule():
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float32)
    rb = np.arange(256, dtype=np.uint8)
    # on the grid: the nearest-even code for every random byte, signs kept
    for sgn in (1, -1):
        t = np.repeat(sgn * grid, 256)
        want = np.repeat(oracle.encode_array(oracle.E2M1, sgn * grid), 256)
        np.testing.assert_array_equal(oracle.e2m1_sr(t, np.tile(rb, 8)), want & 0xF)
    # between grid values: probability of rounding up = floor(256 f) / 256 exactly
    rng = np.random.default_rng(3)
    for _ in range(200):
        i = int(rng.integers(0, 7))
        lo, hi = float(grid[i]), float(grid[i + 1])
        t = np.float32(lo + (hi - lo) * rng.random())
        if t == lo or t >= 6:
            continue
        f = (Fraction(float(t)) - Fraction(lo)) / (Fraction(hi) - Fraction(lo))
        F = int(f * 256)                                            # floor
        codes = oracle.e2m1_sr(np.full(256, t), rb)
        up = codes == oracle.e2m1_sr(np.array([hi], np.float32), np.zeros(1, np.uint8))[0]
        assert int(up.sum()) == F and np.all(up == (rb < F))
        assert oracle.e2m1_sr(np.array([-t]), np.array([0], np.uint8))[0] & 8        # sign kept
    # beyond 6 (and at it): saturate
    np.testing.assert_array_equal(oracle.e2m1_sr(np.array([6, 7, 1e30, -8], np.float32), np.zeros(4, np.uint8)),
                                  np.array([7, 7, 7, 15], np.uint8))


def test_stochastic_rounding_streams_of_the_grouped_cast():
    """ROW_SR / COL_SR: each code is e2m1_sr of its pre-rounding value with
    byte offset + e of the Philox byte stream of seed (rowwise) or seed + 1
    (columnwise; counter = byte / 16 in the two low words), e the element's
    index in its output; block scales and amax as without stochastic
    rounding."""
    x = S.normal_bf16(331, (256, 128))
    splits, mask, seed, offset = [128, 128], 0x3A5C, 0x00FF00FF12345678, 4096
    flags = oracle.ROWWISE | oracle.COLWISE
    rn = oracle.group_rht_quant(x, splits, mask, flags)
    r = oracle.group_rht_quant(x, splits, mask, flags | oracle.ROW_SR | oracle.COL_SR, want_pre=True,
                               seed=seed, offset=offset)
    for k in ("row_sf", "col_sf", "amax_row", "amax_col", "sdec_row", "sdec_col"):
        np.testing.assert_array_equal(r[k], rn[k], err_msg=k)
    n = 256 * 128
    for d, key, pre in ((0, "row_codes", r["row_pre"]), (1, "col_codes", r["col_pre"])):
        k = seed + d
        blocks = [oracle.philox4x32_10([b & 0xFFFFFFFF, b >> 32, 0, 0], [k & 0xFFFFFFFF, k >> 32])
                  for b in range(offset // 16, (offset + n) // 16)]
        rbytes = np.concatenate(blocks).view(np.uint8)                 # little-endian bytes, from byte `offset`
        want = oracle.e2m1_sr(pre.reshape(-1), rbytes)
        np.testing.assert_array_equal(_unpack(r[key]).reshape(-1), want, err_msg=key)
    assert not np.array_equal(r["col_codes"], rn["col_codes"])


def test_nvfp4_zero_section_and_tiny_values():
    x = np.zeros((256, 128), dtype=np.uint16)
    x[128:] = S.normal_bf16(97, (128, 128))
    r = oracle.group_rht_quant(x, [128, 128], 0x00FF)
    assert r["amax_row"][0] == 0 and r["sdec_row"][0] == 1 and r["amax_col"][0] == 0
    assert np.all(r["row_codes"][:128] == 0) and np.all(r["row_sf"][:128] == 0)
    # sigma flips turn +0 into -0, and the sign of zero is kept: every code of
    # the zero section decodes to zero, some of them as -0 (nibble 0x8)
    nib = _unpack(r["col_codes"][: 128 * 128 // 2])
    assert np.all((nib & 7) == 0) and np.any(nib == 8)
    assert np.all(r["col_sf"][: 128 * 128 // 16] == 0)


def _crafted_division_cases(count=24, seed=13):
    """Groups in which q = y / s lands so close to an E4M3 midpoint that
    correctly rounded division and multiplication by a rounded reciprocal pick
    different codes (the one-ulp midpoint cases the onnxruntime PR #33644
    description says its deterministic regressions cover)."""
    rng = np.random.default_rng(seed)
    inv = np.float32(1) / np.float32(448)
    mids = [(lo + hi) / 2 for lo, hi in zip(E4V[:-1], E4V[1:]) if lo >= Fraction(1, 64)]
    cases = []
    while len(cases) < count:
        amax = np.float32(rng.uniform(0.5, 8.0))
        s = amax * inv
        rcp = np.float32(1) / s
        mid = mids[int(rng.integers(len(mids)))]
        y0 = np.float32(float(mid * frac(s)))
        for y in (y0, np.nextafter(y0, np.float32(9)), np.nextafter(y0, np.float32(-9))):
            if not (abs(y) < amax):
                continue
            q_div = np.float32(y) / s                # IEEE binary32 division (numpy)
            q_rcp = np.float32(y) * rcp
            c_div = nearest_code(frac(q_div), E4C, E4V, 0x80, False)
            c_rcp = nearest_code(frac(q_rcp), E4C, E4V, 0x80, False)
            if c_div != c_rcp:
                cases.append((amax, y, c_div))
                break
    return cases


def test_fp8_division_is_correctly_rounded_at_midpoints():
    cases = _crafted_division_cases()
    y = np.zeros((len(cases), 128), dtype=np.float32)
    want = []
    for g, (amax, v, c) in enumerate(cases):
        y[g, 0] = amax
        y[g, 1] = v
        want.append(c)
    codes, scales, _ = oracle.swiglu_fp8_k128(oracle.NONE_F32, y, len(cases), 128)
    assert [int(c) for c in codes[:, 1]] == want
