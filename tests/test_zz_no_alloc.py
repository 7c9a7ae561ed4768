"""GPU: the allocation-free grouped entry point (hq_group_rht_quant_noalloc).

It exists for callers that cannot allocate device memory where they quantize
(frameworks that own all device memory): its scratch
words live in a fixed array inside the library.  Two calls in a row through
the C ABI must give exactly what hq_group_rht_quant gives with a caller
workspace (the parity tests compare outputs bit for bit).  This file is
collected last so that a run stopping at the first failure has run every
other test first; it passes alone in a fresh process as well.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import synthetic as S

pytestmark = pytest.mark.gpu


def _outputs(hq, M, K, nsec):
    return hq.group_outputs(M, K, nsec)


def test_noalloc_matches_workspace_entry_point_twice(hq):
    splits = [256, 0, 128, 384, 128]
    M, K = sum(splits), 384
    x = S.with_outliers_bf16(S.normal_bf16(501, (M, K)), 502, p=0.002)
    xd = torch.from_numpy(x).view(torch.bfloat16).cuda()
    mask = S.sign_mask16(503)
    flags = hq.HQ_ROWWISE | hq.HQ_COLWISE

    ref = _outputs(hq, M, K, len(splits))
    ws = hq.new_workspace(len(splits))
    hq.hq_group_rht_quant(xd, M, K, splits, len(splits), mask, flags, ref["row_codes"], ref["row_sf"],
                          ref["col_codes"], ref["col_sf"], ref["amax_row"], ref["amax_col"], ref["sdec_row"],
                          ref["sdec_col"], ws)
    torch.cuda.synchronize()

    L = hq.lib()
    arr = (ctypes.c_int64 * len(splits))(*splits)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = _outputs(hq, M, K, len(splits))
        for t in out.values():
            t.view(torch.uint8).fill_(0xA5)
        p = lambda k: ctypes.c_void_p(out[k].data_ptr())
        rc = L.hq_group_rht_quant_noalloc(ctypes.c_void_p(xd.data_ptr()), M, K, ctypes.cast(arr, ctypes.c_void_p),
                                          len(splits), mask, flags, p("row_codes"), p("row_sf"), p("col_codes"),
                                          p("col_sf"), p("amax_row"), p("amax_col"), p("sdec_row"), p("sdec_col"),
                                          stream)
        assert rc == hq.HQ_OK, hq.status_string(rc)
        torch.cuda.synchronize()
        for k in ref:
            assert torch.equal(out[k].view(torch.uint8), ref[k].view(torch.uint8)), f"call {call}: {k} differs"


def test_noalloc_rejects_too_many_sections(hq):
    L = hq.lib()
    arr = (ctypes.c_int64 * 257)(*([0] * 257))
    fake = ctypes.c_void_p(0x10000)
    rc = L.hq_group_rht_quant_noalloc(fake, 0, 128, ctypes.cast(arr, ctypes.c_void_p), 257, 0, 3, fake, fake, fake,
                                      fake, fake, fake, fake, fake, None)
    assert rc == hq.HQ_ERR_SHAPE
