"""FORMAT.md against the oracle.

Every constant, code table, layout expression and formula that FORMAT.md
states is parsed from the file and checked here against the oracle on small
inputs: the constants by the oracle's observable results (a scale, an amax),
the layouts and formulas by recomputing the outputs from the document's own
definitions (numpy binary32 arithmetic, stage by stage) and placing them with
the document's offset expressions.  A drift of either the document or the
oracle fails here.
"""
from __future__ import annotations

import os
import re

import numpy as np
import pytest

import oracle
import synthetic as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DOC = open(os.path.join(ROOT, "FORMAT.md"), encoding="utf-8").read()
F = np.float32


# ------------------------------------------------------------------ parsing
def section(title_prefix: str) -> str:
    """Text of the section whose heading starts with `title_prefix`, up to the next heading of any level."""
    m = re.search(r"^#{2,3} " + re.escape(title_prefix) + r".*?$(.*?)(?=^#{2,3} |\Z)", DOC, flags=re.M | re.S)
    assert m, title_prefix
    return m.group(1)


def table_rows(text: str):
    rows = []
    for line in text.splitlines():
        line = line.strip()
        if not line.startswith("|") or set(line) <= set("|-: "):
            continue
        rows.append([c.strip() for c in line.strip("|").split("|")])
    return rows[1:]  # header dropped


def doc_value(s: str) -> float:
    """Value column of the tables: 2^-9, 7·2^-9, RN(1/448), -0, 448 ..."""
    s = s.replace("·", "*").replace("^", "**").replace("−", "-")
    neg = s.startswith("-")
    if neg:
        s = s[1:]
    rn = s.startswith("RN(")
    if rn:
        s = s[3:-1]
    v = float(eval(s, {"__builtins__": {}}))
    v = float(F(v)) if rn else v
    return -v if neg else v


def bits(x) -> int:
    return int(np.array([x], dtype=np.float32).view(np.uint32)[0])


def f32_of(h: int) -> np.float32:
    return np.array([h], dtype=np.uint32).view(np.float32)[0]


def constants():
    out = {}
    for name, hexs, val, *_ in table_rows(section("2. Constants")):
        out[name] = (int(hexs, 16), doc_value(val))
    return out


def layout(sec_prefix: str):
    """{(buffer, element): offset expression (and nibble expression)} of a layout table."""
    out = {}
    for row in table_rows(section(sec_prefix)):
        exprs = re.findall(r"`([^`]*)`", " | ".join(row[2:]))
        out[(row[0], row[1])] = exprs
    return out


def ev(expr: str, **env) -> int:
    return int(eval(expr, {"__builtins__": {}}, env))


# ------------------------------------------------- the document's arithmetic
C = constants()
H16_SCALE, H128_SCALE = f32_of(C["H16_SCALE"][0]), f32_of(C["H128_SCALE"][0])
GNUM, E2MAX = f32_of(C["NVFP4_GLOBAL_NUM"][0]), f32_of(C["E2M1_MAX"][0])
FLOOR, INV448 = f32_of(C["FP8_AMAX_FLOOR"][0]), f32_of(C["FP8_INV448"][0])


def doc_butterfly(v: np.ndarray) -> np.ndarray:
    """Section 3: ascending stages h = 1, 2, ..., n/2 on the last axis (binary32)."""
    v = np.array(v, dtype=np.float32, copy=True)
    n = v.shape[-1]
    h = 1
    while h < n:
        idx = np.array([i for i in range(n) if i & h == 0])
        a, b = v[..., idx].copy(), v[..., idx + h].copy()
        v[..., idx], v[..., idx + h] = a + b, a - b
        h <<= 1
    return v


def doc_rht16(blocks: np.ndarray, mask: int) -> np.ndarray:
    sigma = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(16)], dtype=np.float32)
    return doc_butterfly(blocks * sigma) * H16_SCALE


def doc_global(A: np.float32):
    with np.errstate(divide="ignore", over="ignore", invalid="ignore"):
        s = F(GNUM / F(A))
    if not (A > 0) or not np.isfinite(s):
        s = F(1.0)
    return s, F(F(1.0) / s)


def doc_blocks(v: np.ndarray, S_enc: np.float32):
    """Section 5 per 16-block (last axis 16): (sf codes, pre-rounding values)."""
    ab = np.max(np.abs(v), axis=-1)
    sf = oracle.encode_array(oracle.E4M3, F(ab / E2MAX).astype(np.float32) * S_enc)
    val = np.array([oracle.e4m3_decode(int(c)) for c in sf.reshape(-1)], dtype=np.float32).reshape(sf.shape)
    with np.errstate(divide="ignore"):
        enc = np.where(val == 0, F(0), S_enc / np.where(val == 0, F(1), val)).astype(np.float32)
    return sf, (v * enc[..., None]).astype(np.float32)


def nibble(buf: np.ndarray, off: int, which: int) -> int:
    return (int(buf[off]) >> (4 * which)) & 0xF


# ----------------------------------------------------------------- tables
def test_constants_are_the_stated_values():
    assert len(C) >= 7
    for name, (h, v) in C.items():
        assert bits(v) == h, (name, hex(bits(v)), hex(h))


def test_e4m3_table():
    rows = table_rows(section("1.2 E4M3"))
    assert len(rows) >= 8
    for code, val in rows:
        got = oracle.e4m3_decode(int(code, 16))
        want = doc_value(val)
        assert got == want and np.signbit(F(got)) == np.signbit(F(want)), (code, got, want)
        assert oracle.e4m3_encode(want) == int(code, 16)
    assert oracle.e4m3_encode(1e30) == 0x7E and oracle.e4m3_decode(0x7E) == float(f32_of(C["E4M3_MAX"][0]))
    assert np.isnan(oracle.e4m3_decode(0x7F)) and np.isnan(oracle.e4m3_decode(0xFF))


def test_e2m1_table():
    rows = table_rows(section("1.3 E2M1"))
    seen = {}
    for r in rows:
        for code, val in (r[0:2], r[2:4]):
            seen[int(code, 16)] = doc_value(val)
    assert sorted(seen) == list(range(16))
    for code, want in seen.items():
        got = oracle.e2m1_decode(code)
        assert got == want and np.signbit(F(got)) == np.signbit(F(want)), (code, got, want)
        assert oracle.e2m1_encode(want) == code
    assert oracle.e2m1_encode(100.0) == 7 and oracle.e2m1_decode(7) == float(E2MAX)


# -------------------------------------------------- constants by their role
def test_fp8_scale_constants_by_role():
    x = np.zeros((2, 128), dtype=np.float32)
    x[0, 5] = -1.0  # amax 1
    _, scales, _ = oracle.swiglu_fp8_k128(oracle.NONE_F32, x, 2, 128)
    assert bits(scales[0, 0]) == C["FP8_INV448"][0]
    assert bits(scales[1, 0]) == bits(F(FLOOR * INV448))  # all-zero group: the floor


def test_hadamard_scales_by_role():
    # H128: a unit vector rotates to the constant vector H128_SCALE
    a = np.zeros((1, 1, 128), dtype=np.uint16)
    a[0, 0, 0] = 0x3F80  # 1.0
    _, _, _, amax = oracle.cat_rotate_fp8(a, None, 1, 1, 128, want_amax=True)
    assert bits(amax[0, 0]) == C["H128_SCALE"][0]
    # RHT16: a single 1.0 in a column block gives |v| = H16_SCALE everywhere
    x = np.zeros((128, 128), dtype=np.uint16)
    x[0, 0] = 0x3F80
    r = oracle.group_rht_quant(x, [128], 0, oracle.COLWISE)
    assert bits(r["amax_col"][0]) == C["H16_SCALE"][0]


def test_global_scale_numerator_by_role():
    x = np.zeros((128, 128), dtype=np.uint16)
    x[3, 7] = 0x4040  # 3.0
    r = oracle.group_rht_quant(x, [128], 0, oracle.ROWWISE)
    assert r["amax_row"][0] == 3.0
    assert bits(r["sdec_row"][0]) == bits(F(F(1) / F(GNUM / F(3.0))))


# ------------------------------------------------------------------ layouts
SPLITS = [128, 0, 256]
K = 256


@pytest.fixture(scope="module")
def grouped():
    M = sum(SPLITS)
    x = S.with_outliers_bf16(S.normal_bf16(71, (M, K)), 73, p=0.01, factor=20.0)
    mask = S.sign_mask16(72)
    r = oracle.group_rht_quant(x, SPLITS, mask, oracle.ROWWISE | oracle.COLWISE)
    return x, mask, r


def test_grouped_rowwise_layout_and_formulas(grouped):
    x, mask, r = grouped
    L = layout("6.1")
    off_c, nib_c = L[("row_codes", "(r, k)")]
    (off_s,) = L[("row_sf", "(r, k)")]
    xf = S.bf16_bits_to_f32(x)
    r0 = 0
    for s, Ms in enumerate(SPLITS):
        rows = xf[r0:r0 + Ms]
        A = F(np.max(np.abs(rows))) if Ms else F(0)
        S_enc, sdec = doc_global(A)
        assert bits(r["amax_row"][s]) == bits(A) and bits(r["sdec_row"][s]) == bits(sdec)
        if Ms:
            sf, pre = doc_blocks(rows.reshape(Ms, K // 16, 16), S_enc)
            codes = oracle.encode_array(oracle.E2M1, pre).reshape(Ms, K)
            sf = sf.reshape(Ms, K // 16)
            for rr in range(Ms):
                gr = r0 + rr
                for k in range(0, K, 3):
                    assert nibble(r["row_codes"].reshape(-1), ev(off_c, r=gr, k=k, K=K), ev(nib_c, k=k)) \
                        == codes[rr, k], (s, rr, k)
                    assert r["row_sf"].reshape(-1)[ev(off_s, r=gr, k=k, K=K)] == sf[rr, k // 16]
        r0 += Ms


def test_grouped_columnwise_layout_and_formulas(grouped):
    x, mask, r = grouped
    L = layout("6.1")
    off_c, nib_c = L[("col_codes", "(s, c, m)")]
    (off_s,) = L[("col_sf", "(s, c, m)")]
    xf = S.bf16_bits_to_f32(x)
    r0 = 0
    for s, Ms in enumerate(SPLITS):
        if Ms:
            # [Ms/16, 16, K] -> blocks of 16 consecutive rows of one column: [K, Ms/16, 16]
            blocks = xf[r0:r0 + Ms].reshape(Ms // 16, 16, K).transpose(2, 0, 1)
            v = doc_rht16(blocks, mask)
            A = F(np.max(np.abs(v)))
        else:
            A = F(0)
        S_enc, sdec = doc_global(A)
        assert bits(r["amax_col"][s]) == bits(A) and bits(r["sdec_col"][s]) == bits(sdec)
        if Ms:
            sf, pre = doc_blocks(v, S_enc)
            codes = oracle.encode_array(oracle.E2M1, pre)
            for c in range(0, K, 5):
                for m in range(Ms):
                    o = ev(off_c, K=K, r0=r0, c=c, Ms=Ms, m=m)
                    assert nibble(r["col_codes"], o, ev(nib_c, m=m)) == codes[c, m // 16, m % 16], (s, c, m)
                    assert r["col_sf"][ev(off_s, K=K, r0=r0, c=c, Ms=Ms, m=m)] == sf[c, m // 16]
        r0 += Ms


def test_dsa_layouts_and_fp8_rule():
    M, G, ld = 5, 3, 8
    pe = S.normal_bf16(81, (M, G, 64))
    nope = S.normal_bf16(82, (M, G, 64))
    L = layout("6.2")
    (o_out,) = L[("out_fp8", "(t, g, j)")]
    (o_rm,) = L[("scales, row major", "(t, g)")]
    (o_tr,) = L[("scales, transposed", "(t, g)")]
    o_c4, n_c4 = L[("nvfp4 codes", "(t, g, j)")]
    (o_sf4,) = L[("nvfp4 block_sf", "(t, g, j)")]
    out, sc_rm, _ = oracle.cat_rotate_fp8(pe, nope, M, G, 128)
    out2, sc_tr, _ = oracle.cat_rotate_fp8(pe, nope, M, G, 128, scale_layout=oracle.TRANSPOSED, scale_ld=ld)
    r4 = oracle.cat_rotate_nvfp4(pe, nope, M, G, 128, scale_layout=oracle.TRANSPOSED, scale_ld=ld, want_amax=True)
    assert np.array_equal(out, out2)
    v = np.concatenate([S.bf16_bits_to_f32(pe), S.bf16_bits_to_f32(nope)], axis=-1)  # pe first
    y = doc_butterfly(v) * H128_SCALE
    for t in range(M):
        for g in range(G):
            amax = F(np.max(np.abs(y[t, g])))
            s = F(F(max(amax, FLOOR)) * INV448)
            q = oracle.encode_array(oracle.E4M3, (y[t, g] / s).astype(np.float32))
            assert bits(sc_rm.reshape(-1)[ev(o_rm, t=t, g=g, G=G)]) == bits(s)
            assert bits(sc_tr.reshape(-1)[ev(o_tr, t=t, g=g, ld=ld)]) == bits(s)
            for j in range(128):
                assert out.reshape(-1)[ev(o_out, t=t, g=g, G=G, j=j)] == q[j]
            # FP4: the vector in place of a section
            S_enc, sdec = doc_global(amax)
            assert bits(r4["sdec"].reshape(-1)[ev(o_tr, t=t, g=g, ld=ld)]) == bits(sdec)
            sf, pre = doc_blocks(y[t, g].reshape(8, 16), S_enc)
            codes = oracle.encode_array(oracle.E2M1, pre).reshape(-1)
            for j in range(128):
                assert nibble(r4["codes"].reshape(-1), ev(o_c4, t=t, g=g, G=G, j=j), ev(n_c4, j=j)) == codes[j]
                assert r4["block_sf"].reshape(-1)[ev(o_sf4, t=t, g=g, G=G, j=j)] == sf[j // 16]


def test_k128_layouts_and_swiglu():
    M, K_out = 3, 256
    gu = S.normal_f32(91, (M, 2 * K_out), std=2 ** 0.5)
    L = layout("6.3")
    (o_out,) = L[("out_fp8", "(m, k)")]
    (o_sc,) = L[("scales", "(m, k)")]
    (o_g,) = L[("SwiGLU input gate", "(m, k)")]
    (o_u,) = L[("SwiGLU input up", "(m, k)")]
    out, scales, _ = oracle.swiglu_fp8_k128(oracle.SWIGLU_F32, gu, M, K_out)
    flat = gu.reshape(-1)
    for m in range(M):
        g = np.array([flat[ev(o_g, m=m, k=k, K_out=K_out)] for k in range(K_out)], dtype=np.float32)
        u = np.array([flat[ev(o_u, m=m, k=k, K_out=K_out)] for k in range(K_out)], dtype=np.float32)
        e = oracle.exp_f32(-g)
        act = ((g / (F(1) + e)).astype(np.float32) * u).astype(np.float32)
        for grp in range(K_out // 128):
            y = act[128 * grp:128 * grp + 128]
            s = F(F(max(F(np.max(np.abs(y))), FLOOR)) * INV448)
            q = oracle.encode_array(oracle.E4M3, (y / s).astype(np.float32))
            assert bits(scales.reshape(-1)[ev(o_sc, m=m, k=128 * grp, K_out=K_out)]) == bits(s)
            for j in range(128):
                assert out.reshape(-1)[ev(o_out, m=m, k=128 * grp + j, K_out=K_out)] == q[j]


# ------------------------------------------------------ stochastic rounding
def _doc_philox(ctr, key):
    """Philox4x32-10 from the paper's round function, with FORMAT.md's constants."""
    txt = section("7. Stochastic")
    m0, m1, w0, w1 = (int(h, 16) for h in re.findall(r"0x[0-9A-F]{8}", txt)[:4])
    c = [int(v) for v in ctr]
    k0, k1 = int(key[0]), int(key[1])
    mask = 0xFFFFFFFF
    for rnd in range(10):
        if rnd:
            k0, k1 = (k0 + w0) & mask, (k1 + w1) & mask
        p0, p1 = m0 * c[0], m1 * c[2]
        c = [((p1 >> 32) ^ c[1] ^ k0) & mask, p1 & mask, ((p0 >> 32) ^ c[3] ^ k1) & mask, p0 & mask]
    return c


def _doc_byte(k: int, i: int) -> int:
    w = _doc_philox([(i // 16) & 0xFFFFFFFF, (i // 16) >> 32, 0, 0], [k & 0xFFFFFFFF, k >> 32])
    return (w[(i // 4) % 4] >> (8 * (i % 4))) & 0xFF


def _doc_sr(t: float, r: int) -> int:
    a = abs(float(t))
    sign = 8 if np.signbit(F(t)) else 0
    if not a < 6.0:
        return sign | 7
    step = 0.5 if a < 2 else (1.0 if a < 4 else 2.0)
    n = np.floor(a / step)
    f = a / step - n
    val = (n + (1 if r < int(np.floor(256 * f)) else 0)) * step
    return sign | oracle.e2m1_encode(val)


def test_philox_constants_match_oracle():
    for ctr, key in (([0, 0, 0, 0], [0, 0]), ([1, 2, 3, 4], [5, 6]), ([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2)):
        assert list(oracle.philox4x32_10(ctr, key)) == _doc_philox(ctr, key)


def test_stochastic_rounding_stream_and_rule():
    M, Kk, seed, offset = 128, 128, 0x1234_5678_9ABC, 48
    x = S.normal_bf16(95, (M, Kk))
    mask = S.sign_mask16(96)
    flags = oracle.ROWWISE | oracle.COLWISE | oracle.ROW_SR | oracle.COL_SR
    r = oracle.group_rht_quant(x, [M], mask, flags, want_pre=True, seed=seed, offset=offset)
    L = layout("6.1")
    off_r, nib_r = L[("row_codes", "(r, k)")]
    off_c, nib_c = L[("col_codes", "(s, c, m)")]
    rng = np.random.default_rng(3)
    for _ in range(300):
        rr, k = int(rng.integers(M)), int(rng.integers(Kk))
        e = rr * Kk + k  # index in row_codes' [M, K] element order
        want = _doc_sr(r["row_pre"][rr, k], _doc_byte(seed, offset + e))
        assert nibble(r["row_codes"].reshape(-1), ev(off_r, r=rr, k=k, K=Kk), ev(nib_r, k=k)) == want
        c, m = int(rng.integers(Kk)), int(rng.integers(M))
        o = ev(off_c, K=Kk, r0=0, c=c, Ms=M, m=m)
        e = 2 * o + ev(nib_c, m=m)  # index in col_codes' element order
        want = _doc_sr(r["col_pre"][e], _doc_byte(seed + 1, offset + e))
        assert nibble(r["col_codes"], o, ev(nib_c, m=m)) == want


# ---------------------------------------------------------------- workspace
def test_workspace_size_formula(hq):
    rows = table_rows(section("8. Grouped-call workspace"))
    (expr,) = re.findall(r"`([^`]*)`", dict((r[0], r[1]) for r in rows)["hq_group_rht_quant_workspace_size(S)"])
    for s in (1, 2, 17, 32, 100, 255, 256):
        assert hq.hq_group_rht_quant_workspace_size(s) == ev(expr, S=s)


def test_status_codes(hq):
    txt = section("8. Grouped-call workspace")
    pairs = re.findall(r"(\d) ([A-Z]+)", txt)
    names = {int(n): name for n, name in pairs}
    assert names == {0: "OK", 1: "NULL", 2: "SHAPE", 3: "ALIGN", 4: "WORKSPACE", 5: "UNSUPPORTED", 6: "CUDA",
                     7: "TIMEOUT"}
    for n, name in names.items():
        const = "HQ_OK" if name == "OK" else "HQ_ERR_" + name
        assert getattr(hq, const) == n


# ------------------------------------------------------------- scale formats
def test_ue8m0_bits_expression():
    (expr,) = re.findall(r"`([^`]*)`", " ".join(r[1] for r in table_rows(section("6.4 Scale formats"))[:1]))
    rng = np.random.default_rng(9)
    M, G = 4, 2
    pe = S.normal_bf16(401, (M, G, 64))
    nope = S.with_outliers_bf16(S.normal_bf16(402, (M, G, 64)), 403, p=0.05, factor=300.0)
    _, s_pl, _ = oracle.cat_rotate_fp8(pe, nope, M, G, 128)
    _, s_ue, _ = oracle.cat_rotate_fp8(pe, nope, M, G, 128, scale_layout=oracle.UE8M0)
    vals = list(s_pl.reshape(-1)) + [F(1.0), F(0.75), F(3e38), F(np.inf)] + list(
        (rng.random(200) * np.exp2(rng.integers(-60, 60, 200))).astype(np.float32))
    for v in vals:
        got = ev(expr, bits=lambda x: bits(x), s=F(v)) & 0xFFFFFFFF
        m, e = np.frexp(np.float64(v))
        want = float(v) if (m == 0.5 or not np.isfinite(v)) else float(np.float32(np.ldexp(1.0, int(e))))
        assert float(f32_of(got)) == want, (float(v), hex(got))
    for a, b in zip(s_pl.reshape(-1), s_ue.reshape(-1)):
        assert bits(b) == ev(expr, bits=lambda x: bits(x), s=F(a)) & 0xFFFFFFFF


def test_interleaved_scale_offsets():
    rows = table_rows(section("6.4 Scale formats"))
    (expr,) = re.findall(r"`([^`]*)`", [r for r in rows if r[0] == "interleaved scales"][0][2])
    for R, C in ((128, 8), (256, 16), (384, 28)):
        seen = set()
        for r in range(R):
            for c in range(C):
                o = ev(expr, r=r, c=c, C=C)
                assert o == oracle.sf_swizzled_offset(r, c, C)
                seen.add(o)
        assert seen == set(range(R * C))
