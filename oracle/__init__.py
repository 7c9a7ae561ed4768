"""CPU oracle for the Hadamard-rotation + block-quantization paths.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference leg may import this package.  The product
library (``nvfp4_quantization_group_b200``) never imports it, and it never
imports the product library: the two share no code.

The arithmetic lives in ``hq_oracle.c`` (plain single-threaded C, IEEE
binary32, no contraction); this module compiles it with gcc on first use and
wraps it with numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hq_oracle.c")
_LIB = os.path.join(_HERE, "libhq_oracle.so")
_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile hq_oracle.c into libhq_oracle.so (skipped when up to date)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            i64 = ctypes.c_int64
            L.hqo_e4m3_encode.argtypes = [ctypes.c_float]
            L.hqo_e4m3_encode.restype = ctypes.c_uint8
            L.hqo_e4m3_decode.argtypes = [ctypes.c_uint8]
            L.hqo_e4m3_decode.restype = ctypes.c_float
            L.hqo_e2m1_encode.argtypes = [ctypes.c_float]
            L.hqo_e2m1_encode.restype = ctypes.c_uint8
            L.hqo_e2m1_decode.argtypes = [ctypes.c_uint8]
            L.hqo_e2m1_decode.restype = ctypes.c_float
            L.hqo_encode_array.argtypes = [ctypes.c_int, P, P, i64]
            L.hqo_encode_array.restype = None
            L.hqo_exp.argtypes = [ctypes.c_float]
            L.hqo_exp.restype = ctypes.c_float
            L.hqo_exp_array.argtypes = [P, P, i64]
            L.hqo_exp_array.restype = None
            L.hqo_fwht.argtypes = [P, ctypes.c_int]
            L.hqo_fwht.restype = None
            L.hqo_cat_rotate_fp8.argtypes = [P, i64, ctypes.c_int, P, i64, ctypes.c_int, i64,
                                             ctypes.c_int, ctypes.c_int, P, P, ctypes.c_int, i64, P, P]
            L.hqo_cat_rotate_fp8.restype = ctypes.c_int
            L.hqo_cat_rotate_nvfp4.argtypes = [P, i64, ctypes.c_int, P, i64, ctypes.c_int, i64,
                                               ctypes.c_int, ctypes.c_int, P, P, P, ctypes.c_int, i64, P, P]
            L.hqo_cat_rotate_nvfp4.restype = ctypes.c_int
            L.hqo_swiglu_fp8_k128.argtypes = [ctypes.c_int, P, i64, i64, P, P, P, P]
            L.hqo_swiglu_fp8_k128.restype = ctypes.c_int
            L.hqo_group_rht_quant.argtypes = [P, i64, i64, P, ctypes.c_int, ctypes.c_uint16, ctypes.c_uint,
                                              P, P, P, P, P, P, P, P, P, P]
            L.hqo_group_rht_quant.restype = ctypes.c_int
            u64 = ctypes.c_uint64
            L.hqo_group_rht_quant_sr.argtypes = [P, i64, i64, P, ctypes.c_int, ctypes.c_uint16, ctypes.c_uint,
                                                 u64, u64, P, P, P, P, P, P, P, P, P, P]
            L.hqo_group_rht_quant_sr.restype = ctypes.c_int
            L.hqo_philox4x32_10.argtypes = [P, P, P]
            L.hqo_philox4x32_10.restype = None
            L.hqo_e2m1_sr_array.argtypes = [P, P, P, i64]
            L.hqo_e2m1_sr_array.restype = None
            L.hqo_sf_swizzled_offset.argtypes = [i64, i64, i64]
            L.hqo_sf_swizzled_offset.restype = i64
            _lib = L
    return _lib


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


# ------------------------------------------------------------------ scalars
def e4m3_encode(v: float) -> int:
    return int(lib().hqo_e4m3_encode(float(v)))


def e4m3_decode(c: int) -> float:
    return float(lib().hqo_e4m3_decode(int(c)))


def e2m1_encode(v: float) -> int:
    return int(lib().hqo_e2m1_encode(float(v)))


def e2m1_decode(c: int) -> float:
    return float(lib().hqo_e2m1_decode(int(c)))


E4M3, E2M1 = 0, 1


def encode_array(fmt: int, x: np.ndarray) -> np.ndarray:
    """Per-element E4M3 (fmt 0) or E2M1 nibble (fmt 1) codes of FP32 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().hqo_encode_array(fmt, _ptr(x), _ptr(out), x.size)
    return out


def exp_f32(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty_like(x)
    lib().hqo_exp_array(_ptr(x), _ptr(out), x.size)
    return out


def fwht(v: np.ndarray) -> np.ndarray:
    """Unnormalised Sylvester Hadamard butterfly of an FP32 vector (copy)."""
    v = np.array(v, dtype=np.float32, copy=True)
    lib().hqo_fwht(_ptr(v), v.size)
    return v


# -------------------------------------------------------------- operations
ROWMAJOR, TRANSPOSED = 0, 1
# scale formats: UE8M0 (power-of-two) FP8 scales, added to scale_layout / mode
# of the FP8 calls; interleaved 128 x 4 NVFP4 block-scale tiles, added to the
# grouped cast's flags and to the FP4 DSA call's scale_layout
UE8M0, SF_SWIZZLED = 256, 128


def sf_swizzled_offset(r: int, c: int, cols: int) -> int:
    """Byte of element (r, c) of a [rows, cols] block-scale matrix in the interleaved tiles."""
    return int(lib().hqo_sf_swizzled_offset(r, c, cols))


def cat_rotate_fp8(a, b, M, G, hadamard_n=128, a_row_stride=None, b_row_stride=None,
                   scale_layout=ROWMAJOR, scale_ld=None, want_pre=False, want_amax=False):
    """Concat (a | b) per group, optional 128-point Hadamard, FP8 1x128 quant.

    a, b: uint16 BF16 bit arrays; a_width = a.shape[-1] (b may be None).
    Returns (codes [M, G*128] uint8, scales, pre or None), and with want_amax
    a fourth item: the groups' amax in the scales' layout.
    """
    a = np.ascontiguousarray(a, dtype=np.uint16)
    a_w = int(a.shape[-1])
    a_rs = a_row_stride if a_row_stride is not None else G * a_w
    if b is not None:
        b = np.ascontiguousarray(b, dtype=np.uint16)
        b_w = int(b.shape[-1])
        b_rs = b_row_stride if b_row_stride is not None else G * b_w
    else:
        b_w, b_rs = 0, 0
    out = np.empty((M, G * 128), dtype=np.uint8)
    if (scale_layout & 1) == ROWMAJOR:
        scales = np.empty((M, G), dtype=np.float32)
        ld = G
    else:
        ld = scale_ld if scale_ld is not None else M
        scales = np.zeros((G, ld), dtype=np.float32)
    pre = np.empty((M, G * 128), dtype=np.float32) if want_pre else None
    amax = np.zeros_like(scales) if want_amax else None
    rc = lib().hqo_cat_rotate_fp8(_ptr(a), a_rs, a_w, _ptr(b), b_rs, b_w, M, G, hadamard_n,
                                  _ptr(out), _ptr(scales), scale_layout, ld, _ptr(amax), _ptr(pre))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return (out, scales, pre, amax) if want_amax else (out, scales, pre)


def cat_rotate_nvfp4(a, b, M, G, hadamard_n=128, a_row_stride=None, b_row_stride=None,
                     scale_layout=ROWMAJOR, scale_ld=None, want_pre=False, want_amax=False):
    """Concat (a | b) per group, optional 128-point Hadamard, NVFP4 per
    128-vector (8 blocks of 16, E4M3 block scales, per-vector decode scale).

    Returns a dict: codes [M, G*64] uint8, block_sf [M, G*8] uint8, sdec
    (scales' layout), and amax / pre when asked.
    """
    a = np.ascontiguousarray(a, dtype=np.uint16)
    a_w = int(a.shape[-1])
    a_rs = a_row_stride if a_row_stride is not None else G * a_w
    if b is not None:
        b = np.ascontiguousarray(b, dtype=np.uint16)
        b_w = int(b.shape[-1])
        b_rs = b_row_stride if b_row_stride is not None else G * b_w
    else:
        b_w, b_rs = 0, 0
    r = {"codes": np.empty((M, G * 64), dtype=np.uint8), "block_sf": np.empty((M, G * 8), dtype=np.uint8)}
    if (scale_layout & 1) == ROWMAJOR:
        r["sdec"] = np.empty((M, G), dtype=np.float32)
        ld = G
    else:
        ld = scale_ld if scale_ld is not None else M
        r["sdec"] = np.zeros((G, ld), dtype=np.float32)
    if want_amax:
        r["amax"] = np.zeros_like(r["sdec"])
    if want_pre:
        r["pre"] = np.empty((M, G * 128), dtype=np.float32)
    g = r.get
    rc = lib().hqo_cat_rotate_nvfp4(_ptr(a), a_rs, a_w, _ptr(b), b_rs, b_w, M, G, hadamard_n,
                                    _ptr(r["codes"]), _ptr(r["block_sf"]), _ptr(r["sdec"]), scale_layout, ld,
                                    _ptr(g("amax")), _ptr(g("pre")))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return r


NONE_BF16, NONE_F32, SWIGLU_F32 = 0, 1, 2


def swiglu_fp8_k128(mode, x, M, K_out, want_pre=False, want_amax=False):
    """K128 FP8 quantization of BF16/FP32 rows or of SiLU(gate) * up.

    Returns (codes, scales, pre or None), and with want_amax a fourth item:
    the groups' amax [M, K_out/128]."""
    x = np.ascontiguousarray(x)
    out = np.empty((M, K_out), dtype=np.uint8)
    scales = np.empty((M, K_out // 128), dtype=np.float32)  # (mode may add UE8M0)
    pre = np.empty((M, K_out), dtype=np.float32) if want_pre else None
    amax = np.empty_like(scales) if want_amax else None
    rc = lib().hqo_swiglu_fp8_k128(mode, _ptr(x), M, K_out, _ptr(out), _ptr(scales), _ptr(amax), _ptr(pre))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return (out, scales, pre, amax) if want_amax else (out, scales, pre)


ROWWISE, COLWISE, ROW_RHT, AMAX_GIVEN, ROW_SR, COL_SR = 1, 2, 4, 16, 32, 64  # (+ SF_SWIZZLED)


def e2m1_sr(t, r):
    """Stochastic E2M1 codes of FP32 values t with random bytes r."""
    t = np.ascontiguousarray(t, dtype=np.float32)
    r = np.ascontiguousarray(r, dtype=np.uint8)
    out = np.empty(t.shape, dtype=np.uint8)
    lib().hqo_e2m1_sr_array(_ptr(t), _ptr(r), _ptr(out), t.size)
    return out


def philox4x32_10(ctr, key):
    """Philox4x32-10 of a 4-word counter and a 2-word key -> 4 uint32."""
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.empty(4, dtype=np.uint32)
    lib().hqo_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def group_rht_quant(x, split_rows, sign_mask, flags=ROWWISE | COLWISE, want_pre=False, amax_row=None,
                    amax_col=None, seed=0, offset=0):
    """Grouped RHT16 + NVFP4 cast.  x: uint16 BF16 bits [M, K].

    ROW_RHT (with ROWWISE) rotates every 16-element row block along K before
    the rowwise amax and cast.  ROW_SR / COL_SR round that direction's codes
    stochastically with the random streams of seed / seed + 1 from offset.  AMAX_GIVEN takes the section amax values from
    amax_row / amax_col (float [S]) instead of computing them.

    Returns a dict with row_codes [M, K/2], row_sf [M, K/16], col_codes
    [M*K/2], col_sf [M*K/16] (sections concatenated, each [K, M_s/...]),
    amax_row, amax_col, sdec_row, sdec_col [S] and, if asked, the
    pre-rounding values row_pre [M, K] / col_pre [M*K].
    """
    x = np.ascontiguousarray(x, dtype=np.uint16)
    M, K = x.shape
    splits = np.ascontiguousarray(split_rows, dtype=np.int64)
    S = splits.size
    r = {}
    if flags & ROWWISE:
        r["row_codes"] = np.empty((M, K // 2), dtype=np.uint8)
        r["row_sf"] = np.empty((M, K // 16), dtype=np.uint8)
        r["amax_row"] = np.empty(S, dtype=np.float32)
        r["sdec_row"] = np.empty(S, dtype=np.float32)
        if want_pre:
            r["row_pre"] = np.empty((M, K), dtype=np.float32)
    if flags & COLWISE:
        r["col_codes"] = np.empty(M * K // 2, dtype=np.uint8)
        r["col_sf"] = np.empty(M * K // 16, dtype=np.uint8)
        r["amax_col"] = np.empty(S, dtype=np.float32)
        r["sdec_col"] = np.empty(S, dtype=np.float32)
        if want_pre:
            r["col_pre"] = np.empty(M * K, dtype=np.float32)
    if flags & AMAX_GIVEN:
        if flags & ROWWISE:
            r["amax_row"][:] = np.asarray(amax_row, dtype=np.float32)
        if flags & COLWISE:
            r["amax_col"][:] = np.asarray(amax_col, dtype=np.float32)
    g = r.get
    rc = lib().hqo_group_rht_quant_sr(_ptr(x), M, K, _ptr(splits), S, sign_mask, flags, seed, offset,
                                   _ptr(g("row_codes")), _ptr(g("row_sf")), _ptr(g("col_codes")),
                                   _ptr(g("col_sf")), _ptr(g("amax_row")), _ptr(g("amax_col")),
                                   _ptr(g("sdec_row")), _ptr(g("sdec_col")), _ptr(g("row_pre")),
                                   _ptr(g("col_pre")))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return r
