"""GPU parity: the grouped cast from and to host memory
(hq_group_rht_quant_host), which copies, casts and copies back by groups of
whole sections.  Its outputs must be bit-identical to the device entry on the
same input (itself checked against the oracle), whatever the number of
groups, for every flag set, with page-locked or pageable buffers, and equal
to the oracle on a small case directly."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from _compare import assert_bits_equal, assert_fp4_codes

pytestmark = pytest.mark.gpu


def _case(seed, K, splits):
    M = sum(splits)
    x = S.normal_bf16(seed, (M, K))
    xf = S.bf16_bits_to_f32(x).copy()
    r0 = 0
    for i, m in enumerate(splits):
        xf[r0:r0 + m] *= np.float32(2.0 ** ((i % 5) - 2))
        r0 += m
    return S.with_outliers_bf16(S.f32_to_bf16_bits(xf), seed + 1, p=0.002)


def _device(hq, x, splits, mask, flags, seed=None, offset=0, amax=None):
    M, K = x.shape
    out = hq.group_outputs(M, K, len(splits), flags)
    if amax is not None:
        for k, v in amax.items():
            out[k].copy_(torch.from_numpy(v))
    hq.group_rht_quant(torch.from_numpy(x).view(torch.bfloat16).cuda(), splits, mask, flags, out=out, seed=seed,
                       offset=offset)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in out.items()}


def _host(hq, x, splits, mask, flags, groups=0, pin=True, seed=None, offset=0, amax=None, staging=None):
    M, K = x.shape
    xt = torch.from_numpy(x).view(torch.bfloat16)
    if pin:
        xt = xt.pin_memory()
    out = hq.host_outputs(M, K, len(splits), flags, pin=pin)
    if amax is not None:
        for k, v in amax.items():
            out[k].copy_(torch.from_numpy(v))
    hq.group_rht_quant_host(xt, splits, mask, flags, staging=staging, out=out, groups=groups, seed=seed,
                            offset=offset)
    torch.cuda.current_stream().synchronize()
    return {k: v.numpy().copy() for k, v in out.items()}


def _same(got, want):
    assert set(got) == set(want)
    for k in want:
        assert_bits_equal(got[k].reshape(-1), want[k].reshape(-1), k)


@pytest.mark.parametrize("groups", [1, 2, 3, 0, 32])
def test_host_entry_equals_device_entry_for_any_group_count(hq, groups):
    splits = [128, 0, 256, 128, 0, 384, 128]
    x = _case(601, 256, splits)
    want = _device(hq, x, splits, 0xA5C3, 3)
    _same(_host(hq, x, splits, 0xA5C3, 3, groups=groups), want)


def test_host_entry_matches_oracle(hq):
    splits = [256, 0, 128, 384]
    x = _case(611, 384, splits)
    got = _host(hq, x, splits, 0x3C5A, 3, groups=3)
    want = oracle.group_rht_quant(x, splits, 0x3C5A, 3)
    pre = oracle.group_rht_quant(x, splits, 0x3C5A, 3, want_pre=True)
    for k in ("amax_row", "sdec_row", "row_sf", "amax_col", "sdec_col", "col_sf"):
        assert_bits_equal(got[k].reshape(-1), want[k].reshape(-1), k)
    assert_fp4_codes(got["row_codes"].reshape(want["row_codes"].shape), want["row_codes"], lambda: pre["row_pre"],
                     "row codes")
    assert_fp4_codes(got["col_codes"].reshape(want["col_codes"].shape), want["col_codes"], lambda: pre["col_pre"],
                     "col codes")


@pytest.mark.parametrize("flags", [1, 2, 3 | 4, 3 | 8, 1 | 4, 3 | 128])
def test_host_entry_flags(hq, flags):
    splits = [128, 256, 0, 128]
    x = _case(621, 256, splits)
    _same(_host(hq, x, splits, 0x0FF0, flags, groups=2), _device(hq, x, splits, 0x0FF0, flags))


@pytest.mark.parametrize("flags", [3 | 32 | 64, 1 | 32, 3 | 4 | 64])
def test_host_entry_stochastic_rounding_keeps_the_streams(hq, flags):
    """Each group's random bytes are taken at its elements' own indices, so the
    codes do not depend on the grouping."""
    splits = [128, 128, 256, 0, 128]
    x = _case(631, 256, splits)
    want = _device(hq, x, splits, 0x5555, flags, seed=99, offset=16 * 77)
    for groups in (1, 3, 0):
        _same(_host(hq, x, splits, 0x5555, flags, groups=groups, seed=99, offset=16 * 77), want)


def test_host_entry_amax_given_and_pageable_buffers(hq):
    splits = [256, 128, 128]
    x = _case(641, 256, splits)
    ref = _device(hq, x, splits, 0x1234, 3)
    amax = {"amax_row": ref["amax_row"], "amax_col": ref["amax_col"]}
    given = _device(hq, x, splits, 0x1234, 3 | 16, amax=amax)
    _same(_host(hq, x, splits, 0x1234, 3 | 16, groups=2, amax=amax), given)
    _same(_host(hq, x, splits, 0x1234, 3, groups=2, pin=False), ref)


def test_host_entry_all_sections_empty(hq):
    x = np.zeros((0, 128), dtype=np.uint16)
    got = _host(hq, x, [0, 0, 0], 0x1234, 3)
    assert np.all(got["amax_row"] == 0) and np.all(got["sdec_row"] == 1)
    assert np.all(got["amax_col"] == 0) and np.all(got["sdec_col"] == 1)


def test_host_entry_staging_reused_across_calls(hq):
    """Two calls through one staging buffer: the second call's copies wait
    for the first call's work on the stream."""
    splits = [128, 256]
    x1, x2 = _case(651, 256, splits), _case(652, 256, splits)
    staging = hq.HostStaging(384, 256, 2)
    a = _host(hq, x1, splits, 0x7777, 3, groups=2, staging=staging)
    b = _host(hq, x2, splits, 0x7777, 3, groups=2, staging=staging)
    _same(a, _device(hq, x1, splits, 0x7777, 3))
    _same(b, _device(hq, x2, splits, 0x7777, 3))


@pytest.mark.slow
def test_host_entry_grouped_moe_16384x7168(hq):
    seed = S.SEEDS["grouped_moe"]
    x = S.normal_bf16(seed, (16384, 7168))
    splits = S.moe_splits(seed)
    mask = S.sign_mask16(seed)
    _same(_host(hq, x, splits, mask, 3), _device(hq, x, splits, mask, 3))
