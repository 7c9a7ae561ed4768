"""GPU parity: grouped RHT16 + NVFP4 cast (hq_group_rht_quant) against the
oracle -- small ragged section mixes, both schedules, direction flags,
workspace rest state, repeated calls, guard bands, and the full dense and
grouped-MoE workloads."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from _compare import assert_bits_equal, assert_fp4_codes

pytestmark = pytest.mark.gpu

ROW_KEYS = ("row_codes", "row_sf", "amax_row", "sdec_row")
COL_KEYS = ("col_codes", "col_sf", "amax_col", "sdec_col")
GUARD = 4096


def _bf16_dev(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16).cuda()


def _guarded_outputs(hq, M, K, S, flags):
    """Outputs carved from buffers poisoned with 0xA5 and followed by a guard band."""
    bufs, out = {}, {}
    shapes = {}
    if flags & hq.HQ_ROWWISE:
        shapes.update(row_codes=(M * K // 2, torch.uint8), row_sf=(M * K // 16, torch.uint8),
                      amax_row=(S, torch.float32), sdec_row=(S, torch.float32))
    if flags & hq.HQ_COLWISE:
        shapes.update(col_codes=(M * K // 2, torch.uint8), col_sf=(M * K // 16, torch.uint8),
                      amax_col=(S, torch.float32), sdec_col=(S, torch.float32))
    for k, (n, dt) in shapes.items():
        nbytes = n * (4 if dt == torch.float32 else 1)
        raw = torch.full((nbytes + GUARD,), 0xA5, dtype=torch.uint8, device="cuda")
        bufs[k] = raw
        out[k] = raw[:nbytes].view(dt)
    if "row_codes" in out:
        out["row_codes"] = out["row_codes"].view(M, K // 2)
        out["row_sf"] = out["row_sf"].view(M, K // 16)
    return out, bufs


def _run(hq, x, splits, mask, flags, ws=None):
    M, K = x.shape
    S = len(splits)
    if ws is None:
        ws = hq.new_workspace(S)
    out, bufs = _guarded_outputs(hq, M, K, S, flags)
    hq.group_rht_quant(_bf16_dev(x), splits, mask, flags, ws=ws, out=out)
    torch.cuda.synchronize()
    for k, raw in bufs.items():
        assert torch.all(raw[-GUARD:] == 0xA5), f"guard band of {k} overwritten"
    return {k: v.cpu().numpy() for k, v in out.items()}, ws


def _check(got, want, x, splits, mask, flags):
    pre = {}

    def pre_of(key):
        if key not in pre:
            pre.update(oracle.group_rht_quant(x, splits, mask, flags, want_pre=True))
        return pre[key]

    if flags & oracle.ROWWISE:
        assert_bits_equal(got["amax_row"], want["amax_row"], "amax_row")
        assert_bits_equal(got["sdec_row"], want["sdec_row"], "sdec_row")
        assert_bits_equal(got["row_sf"], want["row_sf"], "row_sf")
        assert_fp4_codes(got["row_codes"], want["row_codes"], lambda: pre_of("row_pre"), "row codes")
    if flags & oracle.COLWISE:
        assert_bits_equal(got["amax_col"], want["amax_col"], "amax_col")
        assert_bits_equal(got["sdec_col"], want["sdec_col"], "sdec_col")
        assert_bits_equal(got["col_sf"], want["col_sf"], "col_sf")
        assert_fp4_codes(got["col_codes"], want["col_codes"], lambda: pre_of("col_pre"), "col codes")


def _case(seed, K, splits, scale_sections=True, outliers=0.002):
    M = sum(splits)
    x = S.normal_bf16(seed, (M, K))
    if scale_sections:
        xf = S.bf16_bits_to_f32(x).copy()
        r0 = 0
        for i, m in enumerate(splits):
            xf[r0:r0 + m] *= np.float32(2.0 ** ((i % 7) - 3))
            r0 += m
        x = S.f32_to_bf16_bits(xf)
    if outliers:
        x = S.with_outliers_bf16(x, seed + 1, p=outliers)
    return x


@pytest.mark.parametrize("flags_extra", [0, 8])
def test_small_sections_both_directions(hq, flags_extra):
    splits = [128, 0, 256, 128, 0, 384]
    x = _case(401, 256, splits)
    mask = 0xA5C3
    flags = hq.HQ_ROWWISE | hq.HQ_COLWISE
    got, _ = _run(hq, x, splits, mask, flags | flags_extra)
    _check(got, oracle.group_rht_quant(x, splits, mask, flags), x, splits, mask, flags)


@pytest.mark.parametrize("flags", [1, 2])
def test_single_direction(hq, flags):
    splits = [256, 128]
    x = _case(411, 384, splits)
    got, _ = _run(hq, x, splits, 0x0F0F, flags)
    _check(got, oracle.group_rht_quant(x, splits, 0x0F0F, flags), x, splits, 0x0F0F, flags)
    assert set(got) == set(ROW_KEYS if flags == 1 else COL_KEYS)


def test_many_sections_random_splits_and_masks(hq):
    splits = S.random_splits(421, total_units=24, sections=40)
    x = _case(422, 512, splits)
    for mask in (0x0000, 0xFFFF, S.sign_mask16(423)):
        got, _ = _run(hq, x, splits, mask, 3)
        _check(got, oracle.group_rht_quant(x, splits, mask, 3), x, splits, mask, 3)


def test_all_sections_empty_and_zero_data(hq):
    splits = [0, 0, 0]
    x = np.zeros((0, 128), dtype=np.uint16)
    got, _ = _run(hq, x, splits, 0x1234, 3)
    assert np.all(got["amax_row"] == 0) and np.all(got["sdec_row"] == 1)
    assert np.all(got["amax_col"] == 0) and np.all(got["sdec_col"] == 1)
    splits = [128, 128]
    x = np.zeros((256, 128), dtype=np.uint16)
    x[128:] = S.normal_bf16(431, (128, 128))
    got, _ = _run(hq, x, splits, 0x00FF, 3)
    _check(got, oracle.group_rht_quant(x, splits, 0x00FF, 3), x, splits, 0x00FF, 3)


def test_workspace_returns_to_rest_and_calls_repeat(hq):
    splits = [128, 256, 0, 128]
    x = _case(441, 256, splits)
    ws = hq.new_workspace(len(splits))
    first, ws = _run(hq, x, splits, 0x5A5A, 3, ws=ws)
    assert torch.count_nonzero(ws).item() == 0, "workspace not back in its rest state"
    for extra in (0, 8, 0):
        again, ws = _run(hq, x, splits, 0x5A5A, 3 | extra, ws=ws)
        for k in first:
            assert_bits_equal(again[k], first[k], k)
        assert torch.count_nonzero(ws).item() == 0
    assert hq.hq_get_error(ws) == 0


def test_extreme_magnitudes(hq):
    splits = [128, 128, 128]
    xf = S.bf16_bits_to_f32(S.normal_bf16(451, (384, 256))).copy()
    xf[:128] *= np.float32(1e-30)      # tiny section
    xf[128:256] *= np.float32(1e30)    # huge section
    xf[256:, :16] = 0.0                # zero blocks inside a normal section
    x = S.f32_to_bf16_bits(xf)
    got, _ = _run(hq, x, splits, 0x8001, 3)
    _check(got, oracle.group_rht_quant(x, splits, 0x8001, 3), x, splits, 0x8001, 3)


@pytest.mark.parametrize("flags", [3 | 8, 1 | 8, 2 | 8])
def test_two_pass_extreme_magnitudes(hq, flags):
    """The two-launch schedule (its amax pass the streaming amax kernel) on
    tiny, huge and zero blocks, each direction alone and both."""
    splits = [128, 0, 128, 128]
    xf = S.bf16_bits_to_f32(S.normal_bf16(461, (384, 384))).copy()
    xf[:128] *= np.float32(1e-30)
    xf[128:256] *= np.float32(1e30)
    xf[256:, :16] = 0.0
    xf[300, 40:56] = -0.0
    x = S.f32_to_bf16_bits(xf)
    base = flags & ~8
    got, ws = _run(hq, x, splits, 0x8001, flags)
    _check(got, oracle.group_rht_quant(x, splits, 0x8001, base), x, splits, 0x8001, base)
    assert torch.count_nonzero(ws).item() == 0


def test_one_large_section_2304x2176(hq):
    """One non-empty section of 306 tiles, at least one wave of the grid: the
    library takes two launches (streaming amax, then the casts) without the
    flag; every output as the oracle, the workspace back at rest."""
    splits = [0, 2304, 0]
    x = _case(471, 2176, splits, outliers=0.001)
    mask = S.sign_mask16(472)
    ws = hq.new_workspace(len(splits))
    for flags in (3, 1, 2, 3 | 128, 7):
        got, ws = _run(hq, x, splits, mask, flags, ws=ws)
        _check(got, oracle.group_rht_quant(x, splits, mask, flags), x, splits, mask, flags)
        assert torch.count_nonzero(ws).item() == 0


@pytest.mark.parametrize("flags", [1 | 4, 1 | 2 | 4, 1 | 2 | 4 | 8])
def test_row_rht_small_sections(hq, flags):
    """Rowwise blocks rotated along K: both schedules, with and without the
    columnwise output."""
    splits = [128, 0, 256, 128, 0, 384]
    x = _case(471, 384, splits)
    mask = 0x9C3A
    base = flags & 7
    got, _ = _run(hq, x, splits, mask, flags)
    _check(got, oracle.group_rht_quant(x, splits, mask, base), x, splits, mask, base)
    if not flags & 2:
        assert set(got) == set(ROW_KEYS)


@pytest.mark.parametrize("factor", [1e-33, 1e-30, 1e30, 1e33])
def test_row_rht_scale_range(hq, factor):
    """Sections on both sides of the range in which 0.25 folds into the
    rotated rows' encode factors, next to a section of zeros."""
    splits = [128, 128, 128]
    xf = S.bf16_bits_to_f32(S.normal_bf16(481, (384, 256))).copy()
    xf[:128] *= np.float32(factor)
    xf[128:256] = 0.0
    xf[256:, 16:32] = 0.0
    x = S.f32_to_bf16_bits(xf)
    got, _ = _run(hq, x, splits, 0x00F1, 7)
    _check(got, oracle.group_rht_quant(x, splits, 0x00F1, 7), x, splits, 0x00F1, 7)


@pytest.mark.slow
def test_dense_nvfp4_8192x4096(hq):
    seed = S.SEEDS["dense_nvfp4"]
    x = S.with_outliers_bf16(S.normal_bf16(seed, (8192, 4096)), seed + 1, p=0.001, factor=50.0)
    mask = S.sign_mask16(seed)
    got, _ = _run(hq, x, [8192], mask, 3)
    _check(got, oracle.group_rht_quant(x, [8192], mask, 3), x, [8192], mask, 3)


@pytest.mark.slow
@pytest.mark.parametrize("flags", [3, 7, 3 | 8])
def test_grouped_moe_16384x7168(hq, flags):
    seed = S.SEEDS["grouped_moe"]
    x = S.normal_bf16(seed, (16384, 7168))
    splits = S.moe_splits(seed)
    mask = S.sign_mask16(seed)
    got, _ = _run(hq, x, splits, mask, flags)
    base = flags & ~8
    _check(got, oracle.group_rht_quant(x, splits, mask, base), x, splits, mask, base)


def _run_given(hq, x, splits, mask, flags, amax_row=None, amax_col=None, ws=None):
    """One call with HQ_AMAX_GIVEN: the amax buffers are filled with the given
    values first and must come back unchanged."""
    M, K = x.shape
    S = len(splits)
    if ws is None:
        ws = hq.new_workspace(S)
    out, bufs = _guarded_outputs(hq, M, K, S, flags)
    if flags & hq.HQ_ROWWISE:
        out["amax_row"].copy_(torch.from_numpy(np.asarray(amax_row, np.float32)))
    if flags & hq.HQ_COLWISE:
        out["amax_col"].copy_(torch.from_numpy(np.asarray(amax_col, np.float32)))
    hq.group_rht_quant(_bf16_dev(x), splits, mask, flags | hq.HQ_AMAX_GIVEN, ws=ws, out=out)
    torch.cuda.synchronize()
    for k, raw in bufs.items():
        assert torch.all(raw[-GUARD:] == 0xA5), f"guard band of {k} overwritten"
    assert torch.count_nonzero(ws).item() == 0, "workspace not back in its rest state"
    got = {k: v.cpu().numpy() for k, v in out.items()}
    if flags & hq.HQ_ROWWISE:
        assert_bits_equal(got["amax_row"], np.asarray(amax_row, np.float32), "given amax_row changed")
    if flags & hq.HQ_COLWISE:
        assert_bits_equal(got["amax_col"], np.asarray(amax_col, np.float32), "given amax_col changed")
    return got


@pytest.mark.parametrize("flags", [3, 1 | 4, 2, 7])
def test_amax_given_equals_two_pass_result(hq, flags):
    """Given the amax the two-pass call computes, the single pass reproduces
    every output of it."""
    splits = [256, 0, 128, 384]
    x = _case(491, 256, splits)
    mask = 0x3C5A
    first, _ = _run(hq, x, splits, mask, flags)
    got = _run_given(hq, x, splits, mask, flags, first.get("amax_row"), first.get("amax_col"))
    for k in first:
        assert_bits_equal(got[k], first[k], k)


def test_amax_given_other_values(hq):
    """Given values other than the data's amax (above, below: saturation,
    zero, negative, NaN, and an empty section) against the oracle."""
    splits = [128, 256, 0, 128, 128]
    x = _case(493, 384, splits)
    mask = 0xF00F
    ref = oracle.group_rht_quant(x, splits, mask, 3)
    ar = ref["amax_row"] * np.float32([2.0, 0.25, 1.0, 1.0, 1.0])
    ac = ref["amax_col"] * np.float32([0.5, 3.0, 1.0, 1.0, 1.0])
    ar[2], ac[2] = 3.0, 0.0                        # empty section
    ar[3], ac[3] = 0.0, -2.0                       # S_enc = 1
    ar[4], ac[4] = np.nan, np.float32(1e-35)       # S_enc = 1; S_enc near FLT_MAX (no 0.25 fold)
    got = _run_given(hq, x, splits, mask, 3, ar, ac)
    want = oracle.group_rht_quant(x, splits, mask, 3 | oracle.AMAX_GIVEN, amax_row=ar, amax_col=ac)
    pre = {}

    def pre_of(key):
        if key not in pre:
            pre.update(oracle.group_rht_quant(x, splits, mask, 3 | oracle.AMAX_GIVEN, want_pre=True,
                                              amax_row=ar, amax_col=ac))
        return pre[key]

    for d in ("row", "col"):
        assert_bits_equal(got[f"sdec_{d}"], want[f"sdec_{d}"], f"sdec_{d}")
        assert_bits_equal(got[f"{d}_sf"], want[f"{d}_sf"], f"{d}_sf")
        assert_fp4_codes(got[f"{d}_codes"], want[f"{d}_codes"], lambda d=d: pre_of(f"{d}_pre"), f"{d} codes")


@pytest.mark.slow
def test_amax_given_grouped_moe_16384x7168(hq):
    seed = S.SEEDS["grouped_moe"]
    x = S.normal_bf16(seed, (16384, 7168))
    splits = S.moe_splits(seed)
    mask = S.sign_mask16(seed)
    want = oracle.group_rht_quant(x, splits, mask, 3)
    got = _run_given(hq, x, splits, mask, 3, want["amax_row"], want["amax_col"])
    _check(got, want, x, splits, mask, 3)


def _run_sr(hq, x, splits, mask, flags, seed, offset):
    M, K = x.shape
    out, bufs = _guarded_outputs(hq, M, K, len(splits), flags)
    ws = hq.new_workspace(len(splits))
    hq.group_rht_quant(_bf16_dev(x), splits, mask, flags, ws=ws, out=out, seed=seed, offset=offset)
    torch.cuda.synchronize()
    for k, raw in bufs.items():
        assert torch.all(raw[-GUARD:] == 0xA5), f"guard band of {k} overwritten"
    assert torch.count_nonzero(ws).item() == 0
    return {k: v.cpu().numpy() for k, v in out.items()}


@pytest.mark.parametrize("flags", [3 | 128, 1 | 4 | 128, 2 | 128, 3 | 8 | 128, 7 | 128])
def test_interleaved_block_scales(hq, flags):
    """row_sf and every section's col_sf block in the interleaved 128 x 4 tiles."""
    splits = [128, 0, 384, 256]
    x = _case(611, 512, splits)
    mask = 0x5A3C
    got, _ = _run(hq, x, splits, mask, flags)
    _check(got, oracle.group_rht_quant(x, splits, mask, flags & ~8), x, splits, mask, flags & ~8)


@pytest.mark.slow
def test_interleaved_block_scales_grouped_moe_16384x7168(hq):
    seed = S.SEEDS["grouped_moe"]
    x = S.normal_bf16(seed, (16384, 7168))
    splits = S.moe_splits(seed)
    mask = S.sign_mask16(seed)
    flags = 3 | hq.HQ_SF_SWIZZLED
    got, _ = _run(hq, x, splits, mask, flags)
    _check(got, oracle.group_rht_quant(x, splits, mask, flags), x, splits, mask, flags)


@pytest.mark.parametrize("flags", [3 | 32 | 64, 1 | 32, 2 | 64, 3 | 64, 1 | 4 | 32, 3 | 4 | 32 | 64 | 8,
                                   3 | 32 | 64 | 128, 3 | 32 | 64 | 8])
def test_stochastic_rounding_matches_oracle(hq, flags):
    """Stochastic rounding is decided by integer comparisons of exact values,
    so the codes must be bit-identical to the oracle's."""
    splits = [128, 0, 256, 128]
    x = _case(501, 384, splits)
    mask, seed, offset = 0x6B2D, 0x0123456789ABCDEF, 16 * 12345
    got = _run_sr(hq, x, splits, mask, flags, seed, offset)
    base = flags & (1 | 2 | 4 | 32 | 64 | 128)
    want = oracle.group_rht_quant(x, splits, mask, base, seed=seed, offset=offset)
    for k in want:
        assert_bits_equal(got[k], want[k], k)


def test_stochastic_rounding_depends_only_on_seed_and_offset(hq):
    splits = [256, 128]
    x = _case(511, 256, splits)
    a = _run_sr(hq, x, splits, 0x1111, 3 | 32 | 64, 5, 0)
    b = _run_sr(hq, x, splits, 0x1111, 3 | 32 | 64 | 8, 5, 0)          # another schedule: same codes
    c = _run_sr(hq, x, splits, 0x1111, 3 | 32 | 64, 6, 0)
    d = _run_sr(hq, x, splits, 0x1111, 3 | 32 | 64, 5, 16)
    for k in a:
        assert_bits_equal(b[k], a[k], k)
    for other in (c, d):
        assert not np.array_equal(other["row_codes"], a["row_codes"])
        assert not np.array_equal(other["col_codes"], a["col_codes"])
        assert_bits_equal(other["row_sf"], a["row_sf"], "row_sf")


@pytest.mark.slow
def test_stochastic_rounding_grouped_moe_16384x7168(hq):
    seed = S.SEEDS["grouped_moe"]
    x = S.normal_bf16(seed, (16384, 7168))
    splits = S.moe_splits(seed)
    mask = S.sign_mask16(seed)
    got = _run_sr(hq, x, splits, mask, 3 | 32 | 64, 2024, 1 << 20)
    want = oracle.group_rht_quant(x, splits, mask, 3 | 32 | 64, seed=2024, offset=1 << 20)
    for k in want:
        assert_bits_equal(got[k], want[k], k)


def test_bounded_wait_reports_timeout_and_recovers(hq):
    """A workspace outside its rest state makes the cast tiles' wait run out:
    one section of 4 column tiles is 4 amax tiles (items 0..3) then 4 cast
    tiles; with the claim counter starting at 1, the first claim (item 0, or
    items 0 and 1 with two tiles per claim) is never made, so the section's
    amax never completes and its cast tiles wait for it.  The call ends by
    itself after the bounded spin, hq_get_error reports HQ_ERR_TIMEOUT, the
    workspace is back at rest and the next call is correct."""
    splits = [128]
    x = _case(461, 512, splits)
    ws = hq.new_workspace(1)
    words = ws.view(torch.int32)
    words[0] = 1                     # claim counter
    out = hq.group_outputs(128, 512, 1)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    hq.group_rht_quant(_bf16_dev(x), splits, 0x1111, 3, ws=ws, out=out)
    t1.record()
    torch.cuda.synchronize()
    assert t0.elapsed_time(t1) < 30000
    assert hq.hq_get_error(ws) == hq.HQ_ERR_TIMEOUT
    assert torch.count_nonzero(ws).item() == 0
    got, _ = _run(hq, x, splits, 0x1111, 3, ws=ws)
    _check(got, oracle.group_rht_quant(x, splits, 0x1111, 3), x, splits, 0x1111, 3)
    assert hq.hq_get_error(ws) == 0
