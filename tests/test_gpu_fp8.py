"""GPU parity: cat -> H128 -> FP8 1x128 (hq_cat_rotate_fp8) and the K128 /
SwiGLU FP8 quantizer (hq_swiglu_fp8_k128) against the oracle, from small
ragged cases to the full DSA-indexer and QMoE workloads."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from _compare import assert_bits_equal, assert_fp8_codes

pytestmark = pytest.mark.gpu


def _dev(a: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if t.dtype == torch.uint16:
        t = t.view(torch.bfloat16)
    return t.cuda()


def _cat_case(hq, pe, nope, M, G, hadamard_n, layout, ld=None):
    a = _dev(pe)
    b = None if nope is None else _dev(nope)
    codes, scales, amax = hq.cat_rotate_fp8(a, b, hadamard_n, layout, ld, want_amax=True)
    torch.cuda.synchronize()
    want_c, want_s, _, want_a = oracle.cat_rotate_fp8(pe, nope, M, G, hadamard_n, scale_layout=layout,
                                                      scale_ld=ld if layout else None, want_amax=True)
    got_s, got_a = scales.cpu().numpy(), amax.cpu().numpy()
    if (layout & 1) == oracle.TRANSPOSED:
        got_s, want_s = got_s[:, :M], want_s[:, :M]
        got_a, want_a = got_a[:, :M], want_a[:, :M]
    assert_bits_equal(got_s, want_s, "scales")
    assert_bits_equal(got_a, want_a, "amax")
    assert_fp8_codes(codes.cpu().numpy(), want_c,
                     lambda: oracle.cat_rotate_fp8(pe, nope, M, G, hadamard_n, scale_layout=layout & oracle.UE8M0,
                                                   want_pre=True)[2])


def test_single_tensor_h128_fp8_512x128(hq):
    x = S.normal_bf16(S.SEEDS["fp8_single"], (512, 1, 128))
    _cat_case(hq, x, None, 512, 1, 128, oracle.ROWMAJOR)


@pytest.mark.parametrize("hadamard_n", [0, 128])
@pytest.mark.parametrize("layout", [0, 1])
def test_cat_ragged_tokens_and_heads(hq, hadamard_n, layout):
    # 37 tokens x 5 heads = 185 vectors: one full tile of 128 and a ragged tail
    M, G = 37, 5
    pe = S.normal_bf16(201, (M, G, 64))
    nope = S.with_outliers_bf16(S.normal_bf16(202, (M, G, 64)), 203, p=0.01)
    _cat_case(hq, pe, nope, M, G, hadamard_n, layout, ld=40 if layout else None)


def test_cat_unequal_widths_and_strided_rows(hq):
    M, G = 50, 3
    big_a = S.normal_bf16(211, (M, G * 32 + 16))        # row stride G*32+16, a_width 32
    big_b = S.normal_bf16(212, (M, G * 96 + 8))         # row stride G*96+8, b_width 96
    a = _dev(big_a)
    b = _dev(big_b)
    codes = torch.empty((M, G * 128), dtype=torch.uint8, device="cuda")
    scales = torch.empty((M, G), dtype=torch.float32, device="cuda")
    hq.hq_cat_rotate_fp8(a, G * 32 + 16, 32, b, G * 96 + 8, 96, M, G, 128, codes, scales, 0, G)
    torch.cuda.synchronize()
    want_c, want_s, _ = oracle.cat_rotate_fp8(big_a[:, : G * 32].reshape(M, G, 32), big_b[:, : G * 96].reshape(M, G, 96),
                                              M, G, 128)
    assert_bits_equal(scales.cpu().numpy(), want_s, "scales")
    assert_fp8_codes(codes.cpu().numpy(), want_c)


@pytest.mark.parametrize("a_width", [8, 40, 96, 120, 128])
def test_cat_split_widths_fp8_and_nvfp4(hq, a_width):
    """pe/nope splits whose 32-element quarter vectors straddle the two inputs
    (8, 40, 120), lie in one of them (96: the 32-byte load path) or have no
    second input (128); both outputs, both scale layouts."""
    M, G = 21, 3
    pe = S.normal_bf16(271 + a_width, (M, G, a_width))
    nope = None if a_width == 128 else \
        S.with_outliers_bf16(S.normal_bf16(272 + a_width, (M, G, 128 - a_width)), 273, p=0.02)
    for layout in (oracle.ROWMAJOR, oracle.TRANSPOSED):
        ld = M + 3 if layout else None
        _cat_case(hq, pe, nope, M, G, 128, layout, ld=ld)
        _cat4_case(hq, pe, nope, M, G, 128, layout, ld=ld)


def test_cat_zero_and_constant_vectors(hq):
    M, G = 3, 2
    pe = np.zeros((M, G, 64), dtype=np.uint16)
    nope = np.zeros((M, G, 64), dtype=np.uint16)
    pe[1] = S.f32_to_bf16_bits(np.full((G, 64), 1.5, np.float32))
    nope[2, 1, 7] = S.f32_to_bf16_bits(np.float32([-3.0]))[0]
    _cat_case(hq, pe, nope, M, G, 128, oracle.ROWMAJOR)
    _cat_case(hq, pe, nope, M, G, 0, oracle.ROWMAJOR)


@pytest.mark.parametrize("hadamard_n", [0, 128])
@pytest.mark.parametrize("layout", [0, 1])
def test_cat_ue8m0_ragged_tokens_and_heads(hq, hadamard_n, layout):
    """UE8M0 scales: powers of two, codes of y / 2^k."""
    M, G = 37, 5
    pe = S.normal_bf16(221, (M, G, 64))
    nope = S.with_outliers_bf16(S.normal_bf16(222, (M, G, 64)), 223, p=0.01, factor=1e3)
    _cat_case(hq, pe, nope, M, G, hadamard_n, layout | hq.HQ_FP8_UE8M0, ld=40 if layout else None)


@pytest.mark.slow
def test_dsa_indexer_ue8m0_full_4096x64(hq):
    seed = S.SEEDS["dsa_indexer"]
    pe = S.normal_bf16(seed, (4096, 64, 64))
    nope = S.normal_bf16(seed + 100, (4096, 64, 64))
    _cat_case(hq, pe, nope, 4096, 64, 128, oracle.TRANSPOSED | hq.HQ_FP8_UE8M0, ld=4096)


@pytest.mark.slow
def test_dsa_indexer_full_4096x64(hq):
    """Full DSA indexer prep: q_pe, q_nope [4096, 64, 64], transposed scales [64, 4096]."""
    seed = S.SEEDS["dsa_indexer"]
    pe = S.normal_bf16(seed, (4096, 64, 64))
    nope = S.normal_bf16(seed + 100, (4096, 64, 64))
    _cat_case(hq, pe, nope, 4096, 64, 128, oracle.TRANSPOSED, ld=4096)


# ------------------------------------------------------- cat -> H128 -> NVFP4
from _compare import assert_fp4_codes  # noqa: E402


def _cat4_case(hq, pe, nope, M, G, hadamard_n, layout, ld=None):
    a = _dev(pe)
    b = None if nope is None else _dev(nope)
    got = hq.cat_rotate_nvfp4(a, b, hadamard_n, layout, ld, want_amax=True)
    torch.cuda.synchronize()
    got = {k: v.cpu().numpy() for k, v in got.items()}
    want = oracle.cat_rotate_nvfp4(pe, nope, M, G, hadamard_n, scale_layout=layout,
                                   scale_ld=ld if layout else None, want_amax=True)
    for k in ("sdec", "amax"):
        g, w = got[k], want[k]
        if (layout & 1) == oracle.TRANSPOSED:
            g, w = g[:, :M], w[:, :M]
        assert_bits_equal(g, w, k)
    assert_bits_equal(got["block_sf"], want["block_sf"], "block_sf")
    assert_fp4_codes(got["codes"], want["codes"],
                     lambda: oracle.cat_rotate_nvfp4(pe, nope, M, G, hadamard_n, want_pre=True)["pre"], "fp4 codes")


@pytest.mark.parametrize("hadamard_n", [0, 128])
@pytest.mark.parametrize("layout", [0, 1])
def test_cat_nvfp4_ragged_tokens_and_heads(hq, hadamard_n, layout):
    M, G = 37, 5
    pe = S.normal_bf16(241, (M, G, 64))
    nope = S.with_outliers_bf16(S.normal_bf16(242, (M, G, 64)), 243, p=0.01)
    _cat4_case(hq, pe, nope, M, G, hadamard_n, layout, ld=40 if layout else None)


def test_cat_nvfp4_zero_constant_and_single_tensor(hq):
    M, G = 3, 2
    pe = np.zeros((M, G, 64), dtype=np.uint16)
    nope = np.zeros((M, G, 64), dtype=np.uint16)
    pe[1] = S.f32_to_bf16_bits(np.full((G, 64), 1.5, np.float32))
    nope[2, 1, 7] = S.f32_to_bf16_bits(np.float32([-3.0]))[0]
    _cat4_case(hq, pe, nope, M, G, 128, oracle.ROWMAJOR)
    _cat4_case(hq, pe, nope, M, G, 0, oracle.ROWMAJOR)
    x = S.normal_bf16(251, (512, 1, 128))
    _cat4_case(hq, x, None, 512, 1, 128, oracle.ROWMAJOR)


def test_cat_nvfp4_magnitudes(hq):
    """Vectors from 1e-30 to 1e30 (the slow encode path near the ends)."""
    M, G = 8, 4
    xf = S.bf16_bits_to_f32(S.normal_bf16(261, (M, G, 128))).copy()
    xf *= np.float32(10.0) ** np.arange(-30, 34, 8, dtype=np.float32)[:, None, None]
    x = S.f32_to_bf16_bits(xf)
    _cat4_case(hq, x[..., :64].copy(), x[..., 64:].copy(), M, G, 128, oracle.TRANSPOSED, ld=8)


@pytest.mark.parametrize("layout", [0, 1])
def test_cat_nvfp4_interleaved_block_scales(hq, layout):
    """Block scales in the interleaved 128 x 4 tiles (M a multiple of 128)."""
    M, G = 256, 3
    pe = S.normal_bf16(271, (M, G, 64))
    nope = S.with_outliers_bf16(S.normal_bf16(272, (M, G, 64)), 273, p=0.01)
    _cat4_case(hq, pe, nope, M, G, 128, layout | hq.HQ_SF_SWIZZLED, ld=264 if layout else None)


@pytest.mark.slow
def test_dsa_indexer_nvfp4_interleaved_full_4096x64(hq):
    seed = S.SEEDS["dsa_indexer"]
    pe = S.normal_bf16(seed, (4096, 64, 64))
    nope = S.normal_bf16(seed + 100, (4096, 64, 64))
    _cat4_case(hq, pe, nope, 4096, 64, 128, oracle.TRANSPOSED | hq.HQ_SF_SWIZZLED, ld=4096)


@pytest.mark.slow
def test_dsa_indexer_nvfp4_full_4096x64(hq):
    seed = S.SEEDS["dsa_indexer"]
    pe = S.normal_bf16(seed, (4096, 64, 64))
    nope = S.normal_bf16(seed + 100, (4096, 64, 64))
    _cat4_case(hq, pe, nope, 4096, 64, 128, oracle.TRANSPOSED, ld=4096)


# ------------------------------------------------------------------ K128
def _k128_case(hq, mode, x, M, K_out):
    codes, scales, amax = hq.swiglu_fp8_k128(mode, _dev(x), K_out, want_amax=True)
    torch.cuda.synchronize()
    want_c, want_s, _, want_a = oracle.swiglu_fp8_k128(mode, x, M, K_out, want_amax=True)
    assert_bits_equal(scales.cpu().numpy(), want_s, "scales")
    assert_bits_equal(amax.cpu().numpy(), want_a, "amax")
    assert_fp8_codes(codes.cpu().numpy(), want_c, lambda: oracle.swiglu_fp8_k128(mode, x, M, K_out, True)[2])


@pytest.mark.parametrize("M,K", [(1, 128), (3, 384), (33, 1152), (130, 256)])
def test_k128_bf16_ragged(hq, M, K):
    x = S.with_outliers_bf16(S.normal_bf16(301 + M, (M, K)), 302, p=0.01)
    _k128_case(hq, hq.HQ_ACT_NONE_BF16, x, M, K)


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_k128_ue8m0_all_modes(hq, mode):
    M, K = 33, 640
    if mode == 0:
        x = S.with_outliers_bf16(S.normal_bf16(341, (M, K)), 342, p=0.01, factor=1e4)
    elif mode == 1:
        x = S.normal_f32(343, (M, K), std=3.0)
        x[0, :4] = [0.0, -0.0, 1e-30, 448.0]
        x[1] = 0.0
    else:
        x = S.normal_f32(344, (M, 2 * K), std=2 ** 0.5)
    _k128_case(hq, mode | hq.HQ_FP8_UE8M0, x, M, K)


@pytest.mark.parametrize("M,K", [(1, 128), (7, 640), (65, 256)])
def test_k128_f32_ragged(hq, M, K):
    x = S.normal_f32(311 + M, (M, K), std=3.0)
    x[0, :5] = [0.0, -0.0, 1e-30, -1e-38, 65504.0 * 8]
    _k128_case(hq, hq.HQ_ACT_NONE_F32, x, M, K)


@pytest.mark.parametrize("M,K", [(1, 128), (9, 384), (64, 2048)])
def test_swiglu_ragged(hq, M, K):
    x = S.normal_f32(321 + M, (M, 2 * K), std=math.sqrt(2.0))
    x[0, :4] = [0.0, -0.0, 95.0, -120.0]          # exp overflow/underflow branches
    x[0, K:K + 4] = [1.0, 2.0, 3.0, -4.0]
    _k128_case(hq, hq.HQ_ACT_SWIGLU_F32, x, M, K)


def test_swiglu_exp_sweep_against_oracle(hq):
    """SiLU(g) * 1 over a dense sweep of g: the device exp / division sequence
    reproduces the oracle's bit for bit (checked through the codes and scales
    of single-value groups with a fixed amax)."""
    g = np.linspace(-110.0, 95.0, 127 * 4000, dtype=np.float32)
    M = g.size // 127
    x = np.zeros((M, 256), dtype=np.float32)
    x[:, 1:128] = g.reshape(M, 127)
    x[:, 0] = 200.0                 # silu(200) = 200: fixes amax
    x[:, 128:] = 1.0                # up = 1
    _k128_case(hq, hq.HQ_ACT_SWIGLU_F32, x, M, 128)


def test_k128_nan_and_inf_groups(hq):
    x = S.normal_f32(331, (2, 128))
    x[0, 3] = np.nan
    x[1, 4] = np.inf
    codes, scales, amax = hq.swiglu_fp8_k128(hq.HQ_ACT_NONE_F32, _dev(x), 128, want_amax=True)
    want_c, want_s, _, want_a = oracle.swiglu_fp8_k128(oracle.NONE_F32, x, 2, 128, want_amax=True)
    assert_bits_equal(scales.cpu().numpy(), want_s, "scales")
    assert_bits_equal(amax.cpu().numpy(), want_a, "amax")
    assert_fp8_codes(codes.cpu().numpy(), want_c)
    assert (codes[0, 3].item() & 0x7F) == 0x7F


@pytest.mark.slow
def test_qmoe_full_bf16_32768x4096(hq):
    x = S.normal_bf16(S.SEEDS["qmoe"], (32768, 4096))
    _k128_case(hq, hq.HQ_ACT_NONE_BF16, x, 32768, 4096)


@pytest.mark.slow
def test_qmoe_full_swiglu_32768x2048(hq):
    x = S.normal_f32(S.SEEDS["qmoe"] + 100, (32768, 4096), std=math.sqrt(2.0))
    _k128_case(hq, hq.HQ_ACT_SWIGLU_F32, x, 32768, 2048)
