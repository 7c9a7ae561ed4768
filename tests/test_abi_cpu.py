"""Host-side checks of the C ABI (no GPU needed).

The library must load, export every function include/hq.h declares, and
reject bad arguments with the documented status before touching the GPU.
Pointers here are fake non-null addresses: every call below fails argument
checks, so nothing is dereferenced or launched.
"""
from __future__ import annotations

import ctypes
import os
import re

import pytest

import nvfp4_quantization_group_b200 as hq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hq.h")
FAKE = 0x10000  # 16-byte aligned, never dereferenced
P = ctypes.c_void_p


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hq_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    return hq.lib()


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(hq.EXPORTED)


def test_version_and_status_strings(L):
    assert hq.hq_version() >= 1
    for s in range(8):
        assert hq.status_string(s)
    assert hq.status_string(hq.HQ_ERR_ALIGN).startswith("misaligned")


def test_workspace_size_query():
    assert hq.hq_group_rht_quant_workspace_size(0) == 0
    assert hq.hq_group_rht_quant_workspace_size(hq.HQ_MAX_SECTIONS + 1) == 0
    s1 = hq.hq_group_rht_quant_workspace_size(1)
    s32 = hq.hq_group_rht_quant_workspace_size(32)
    s256 = hq.hq_group_rht_quant_workspace_size(256)
    assert s256 == 3328                     # the noalloc scratch array is sized to this
    assert s1 >= 4 and s1 % 256 == 0 and s1 <= s32 <= s256
    assert s32 >= 4 * (4 + 3 * 32)          # counter word first, then per-section words


def _grp(L, x=FAKE, M=256, K=256, splits=(128, 128), flags=3, ptrs=FAKE, ws=FAKE, ws_bytes=4096,
         row_codes=None):
    arr = (ctypes.c_int64 * len(splits))(*splits)
    rc = FAKE if row_codes is None else row_codes
    return L.hq_group_rht_quant(P(x), M, K, ctypes.cast(arr, P), len(splits), 0x1234, flags,
                                P(rc), P(ptrs), P(ptrs), P(ptrs), P(ptrs), P(ptrs), P(ptrs), P(ptrs),
                                P(ws), ws_bytes, None)


def test_group_rht_quant_argument_errors(L):
    assert _grp(L, flags=0) == hq.HQ_ERR_UNSUPPORTED
    assert _grp(L, flags=16) == hq.HQ_ERR_UNSUPPORTED
    assert _grp(L, flags=hq.HQ_COLWISE | hq.HQ_ROW_RHT) == hq.HQ_ERR_UNSUPPORTED  # rotation without rows
    assert _grp(L, flags=3 | hq.HQ_COL_SR) == hq.HQ_ERR_UNSUPPORTED               # needs the _sr entry (a seed)


def _grp_sr(L, flags=3 | 32 | 64, offset=0, seed=7):
    arr = (ctypes.c_int64 * 2)(128, 128)
    return L.hq_group_rht_quant_sr(P(FAKE), 256, 256, ctypes.cast(arr, P), 2, 0x1234, flags, seed, offset,
                                   P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE),
                                   P(FAKE), 4096, None)


def test_group_rht_quant_sr_argument_errors(L):
    assert _grp_sr(L, offset=8) == hq.HQ_ERR_ALIGN                        # offset % 16
    assert _grp_sr(L, flags=hq.HQ_COLWISE | hq.HQ_ROW_SR) == hq.HQ_ERR_UNSUPPORTED
    assert _grp_sr(L, flags=hq.HQ_ROWWISE | hq.HQ_COL_SR) == hq.HQ_ERR_UNSUPPORTED
    assert _grp_sr(L, flags=3 | 512) == hq.HQ_ERR_UNSUPPORTED
    assert _grp(L, x=0) == hq.HQ_ERR_NULL
    assert _grp(L, ws=0) == hq.HQ_ERR_NULL
    assert _grp(L, ptrs=0) == hq.HQ_ERR_NULL
    assert _grp(L, K=200) == hq.HQ_ERR_ALIGN                       # K % 128
    assert _grp(L, splits=(64, 192)) == hq.HQ_ERR_ALIGN            # split % 128 (fusion rule)
    assert _grp(L, splits=(128, 256)) == hq.HQ_ERR_SHAPE           # sum != M
    assert _grp(L, splits=(128, -128, 256)) == hq.HQ_ERR_SHAPE
    assert _grp(L, splits=(128,) * 2 + (0,) * 300, M=256) == hq.HQ_ERR_SHAPE  # S > 256
    assert _grp(L, ws_bytes=16) == hq.HQ_ERR_WORKSPACE
    assert _grp(L, x=FAKE + 8) == hq.HQ_ERR_ALIGN
    assert _grp(L, row_codes=FAKE + 4) == hq.HQ_ERR_ALIGN


def _grp_host(L, flags=3, M=256, K=256, splits=(128, 128), x=FAKE, ptrs=FAKE, dev=0x100000, dev_bytes=None,
              groups=0, streams=(1, 2, 3), offset=0, split_ptr=True):
    arr = (ctypes.c_int64 * len(splits))(*splits)
    nbytes = hq.hq_group_rht_quant_host_device_bytes(M, K, len(splits)) if dev_bytes is None else dev_bytes
    return L.hq_group_rht_quant_host(P(x), M, K, ctypes.cast(arr, P) if split_ptr else None, len(splits), 0x1234,
                                     flags, 7, offset, P(ptrs), P(ptrs), P(ptrs), P(ptrs), P(ptrs), P(ptrs),
                                     P(ptrs), P(ptrs), P(dev), nbytes, groups, P(streams[0]), P(streams[1]),
                                     P(streams[2]))


def test_group_rht_quant_host_sizes_and_argument_errors(L):
    # staging: x + codes + scales of both directions + 4 section arrays + workspace, 256-byte pieces
    n = hq.hq_group_rht_quant_host_device_bytes(256, 256, 2)
    e = 256 * 256
    assert n >= 2 * e + 2 * (e // 2 + e // 16) + hq.hq_group_rht_quant_workspace_size(2) and n % 256 == 0
    assert hq.hq_group_rht_quant_host_device_bytes(256, 200, 2) == 0        # K % 128
    assert hq.hq_group_rht_quant_host_device_bytes(256, 256, 0) == 0
    assert hq.hq_group_rht_quant_host_device_bytes(-1, 256, 1) == 0
    assert _grp_host(L, flags=0) == hq.HQ_ERR_UNSUPPORTED
    assert _grp_host(L, flags=3 | 512) == hq.HQ_ERR_UNSUPPORTED
    assert _grp_host(L, flags=hq.HQ_COLWISE | hq.HQ_ROW_SR) == hq.HQ_ERR_UNSUPPORTED
    assert _grp_host(L, flags=3 | hq.HQ_COL_SR, offset=8) == hq.HQ_ERR_ALIGN
    assert _grp_host(L, split_ptr=False) == hq.HQ_ERR_NULL
    assert _grp_host(L, dev=0) == hq.HQ_ERR_NULL
    assert _grp_host(L, x=0) == hq.HQ_ERR_NULL
    assert _grp_host(L, ptrs=0) == hq.HQ_ERR_NULL
    assert _grp_host(L, K=200) == hq.HQ_ERR_ALIGN
    assert _grp_host(L, splits=(128, 256)) == hq.HQ_ERR_SHAPE
    assert _grp_host(L, splits=(64, 192)) == hq.HQ_ERR_ALIGN
    assert _grp_host(L, dev=0x100000 + 16) == hq.HQ_ERR_ALIGN               # staging 256-byte aligned
    assert _grp_host(L, dev_bytes=n - 1) == hq.HQ_ERR_WORKSPACE
    assert _grp_host(L, groups=hq.HQ_HOST_MAX_GROUPS + 1) == hq.HQ_ERR_UNSUPPORTED
    assert _grp_host(L, groups=-1) == hq.HQ_ERR_UNSUPPORTED
    assert _grp_host(L, streams=(1, 2, 2)) == hq.HQ_ERR_UNSUPPORTED         # copy streams must differ
    assert _grp_host(L, streams=(1, 1, 3)) == hq.HQ_ERR_UNSUPPORTED


def test_host_wrapper_needs_a_seed_for_stochastic_rounding():
    import torch
    x = torch.zeros((128, 128), dtype=torch.bfloat16)
    with pytest.raises(hq.HQError):
        hq.group_rht_quant_host(x, [128], 0x1234, hq.HQ_ROWWISE | hq.HQ_ROW_SR)


def test_cat_rotate_fp8_argument_errors(L):
    def call(a=FAKE, a_rs=64 * 64, aw=64, b=FAKE, b_rs=64 * 64, bw=64, M=16, G=64, hn=128, out=FAKE,
             sc=FAKE, layout=0, ld=16, amax=None):
        return L.hq_cat_rotate_fp8(P(a), a_rs, aw, P(b), b_rs, bw, M, G, hn, P(out), P(sc), layout, ld,
                                   P(amax), None, 0, None)
    assert call(hn=64) == hq.HQ_ERR_UNSUPPORTED
    assert call(layout=2) == hq.HQ_ERR_UNSUPPORTED
    assert call(aw=64, bw=32) == hq.HQ_ERR_SHAPE                  # widths must sum to 128
    assert call(M=0) == hq.HQ_OK                                   # empty: nothing to do
    assert call(a=0) == hq.HQ_ERR_NULL
    assert call(b=0) == hq.HQ_ERR_NULL
    assert call(aw=60, bw=68) == hq.HQ_ERR_ALIGN
    assert call(a_rs=64 * 64 + 4) == hq.HQ_ERR_ALIGN
    assert call(a_rs=64) == hq.HQ_ERR_SHAPE                        # stride shorter than G groups
    assert call(layout=1, ld=8) == hq.HQ_ERR_SHAPE                 # transposed ld < M
    assert call(out=FAKE + 1) == hq.HQ_ERR_ALIGN
    assert call(amax=FAKE + 2) == hq.HQ_ERR_ALIGN
    assert call(layout=hq.HQ_SF_SWIZZLED) == hq.HQ_ERR_UNSUPPORTED   # a format bit of the FP4 call
    assert call(layout=1 | hq.HQ_FP8_UE8M0, ld=8) == hq.HQ_ERR_SHAPE  # UE8M0 keeps the layout's checks
    assert L.hq_cat_rotate_fp8_workspace_size() == 0


def test_cat_rotate_nvfp4_argument_errors(L):
    def call(a=FAKE, a_rs=64 * 64, aw=64, b=FAKE, b_rs=64 * 64, bw=64, M=16, G=64, hn=128, codes=FAKE, sf=FAKE,
             sc=FAKE, layout=0, ld=16, amax=None):
        return L.hq_cat_rotate_nvfp4(P(a), a_rs, aw, P(b), b_rs, bw, M, G, hn, P(codes), P(sf), P(sc), layout, ld,
                                     P(amax), None, 0, None)
    assert call(hn=16) == hq.HQ_ERR_UNSUPPORTED
    assert call(layout=3) == hq.HQ_ERR_UNSUPPORTED
    assert call(aw=64, bw=16) == hq.HQ_ERR_SHAPE
    assert call(M=0) == hq.HQ_OK
    assert call(sf=0) == hq.HQ_ERR_NULL
    assert call(codes=0) == hq.HQ_ERR_NULL
    assert call(sc=0) == hq.HQ_ERR_NULL
    assert call(codes=FAKE + 8) == hq.HQ_ERR_ALIGN
    assert call(amax=FAKE + 2) == hq.HQ_ERR_ALIGN
    assert call(layout=1, ld=8) == hq.HQ_ERR_SHAPE
    assert call(layout=hq.HQ_FP8_UE8M0) == hq.HQ_ERR_UNSUPPORTED     # a format bit of the FP8 calls
    assert call(layout=hq.HQ_SF_SWIZZLED) == hq.HQ_ERR_ALIGN         # interleaved tiles need M % 128 == 0
    assert L.hq_cat_rotate_nvfp4_workspace_size() == 0


def test_swiglu_fp8_k128_argument_errors(L):
    def call(mode=0, inp=FAKE, M=4, K=256, out=FAKE, sc=FAKE, amax=None):
        return L.hq_swiglu_fp8_k128(mode, P(inp), M, K, P(out), P(sc), P(amax), None, 0, None)
    assert call(mode=3) == hq.HQ_ERR_UNSUPPORTED
    assert call(mode=3 | hq.HQ_FP8_UE8M0) == hq.HQ_ERR_UNSUPPORTED
    assert call(mode=hq.HQ_SF_SWIZZLED) == hq.HQ_ERR_UNSUPPORTED
    assert call(mode=hq.HQ_FP8_UE8M0, K=200) == hq.HQ_ERR_ALIGN
    assert call(K=200) == hq.HQ_ERR_ALIGN
    assert call(M=-1) == hq.HQ_ERR_SHAPE
    assert call(M=0) == hq.HQ_OK
    assert call(inp=0) == hq.HQ_ERR_NULL
    assert call(inp=FAKE + 8) == hq.HQ_ERR_ALIGN
    assert call(sc=FAKE + 2) == hq.HQ_ERR_ALIGN
    assert call(amax=FAKE + 1) == hq.HQ_ERR_ALIGN
    assert L.hq_swiglu_fp8_k128_workspace_size() == 0


def test_convert_and_workspace_argument_errors(L):
    assert L.hq_convert(2, P(FAKE), P(FAKE), 10, None) == hq.HQ_ERR_UNSUPPORTED
    assert L.hq_convert(0, P(FAKE), P(FAKE), -1, None) == hq.HQ_ERR_SHAPE
    assert L.hq_convert(0, P(FAKE), P(FAKE), 0, None) == hq.HQ_OK
    assert L.hq_convert(0, None, P(FAKE), 10, None) == hq.HQ_ERR_NULL
    assert L.hq_convert_e2m1_sr(P(FAKE), P(FAKE), P(FAKE), -1, None) == hq.HQ_ERR_SHAPE
    assert L.hq_convert_e2m1_sr(P(FAKE), P(FAKE), P(FAKE), 0, None) == hq.HQ_OK
    assert L.hq_convert_e2m1_sr(P(FAKE), None, P(FAKE), 10, None) == hq.HQ_ERR_NULL
    assert L.hq_convert_e2m1_sr(None, P(FAKE), P(FAKE), 10, None) == hq.HQ_ERR_NULL
    assert L.hq_workspace_init(None, 256, None) == hq.HQ_ERR_NULL
    assert L.hq_workspace_init(P(FAKE + 4), 256, None) == hq.HQ_ERR_ALIGN
    err = ctypes.c_uint32(0)
    assert L.hq_get_error(None, 256, ctypes.byref(err), None) == hq.HQ_ERR_NULL
    assert L.hq_get_error(P(FAKE), 8, ctypes.byref(err), None) == hq.HQ_ERR_WORKSPACE
