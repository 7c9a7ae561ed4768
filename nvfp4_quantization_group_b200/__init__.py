"""Python binding of the hq C ABI (include/hq.h): argument marshalling only.

Every function below passes raw device pointers and sizes to the compiled
library ``libhq.so`` (CUDA kernels for sm_100a); no step of the computation
runs in Python or PyTorch.  PyTorch is used for device memory and streams.
If the library is missing or fails to load, importing the compute functions
raises: there is no fallback.

Low-level calls (``hq_*``) take caller-allocated output tensors exactly like
the C functions.  ``group_rht_quant``, ``cat_rotate_fp8`` and
``swiglu_fp8_k128`` allocate the outputs with torch and call them.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhq.so")

HQ_OK, HQ_ERR_NULL, HQ_ERR_SHAPE, HQ_ERR_ALIGN, HQ_ERR_WORKSPACE, HQ_ERR_UNSUPPORTED, HQ_ERR_CUDA, \
    HQ_ERR_TIMEOUT = range(8)
HQ_ROWWISE, HQ_COLWISE, HQ_ROW_RHT, HQ_TWO_PASS, HQ_AMAX_GIVEN, HQ_ROW_SR, HQ_COL_SR = 1, 2, 4, 8, 16, 32, 64
HQ_SCALE_ROWMAJOR, HQ_SCALE_TRANSPOSED = 0, 1
HQ_SF_SWIZZLED, HQ_FP8_UE8M0 = 128, 256  # scale formats (see include/hq.h)
HQ_ACT_NONE_BF16, HQ_ACT_NONE_F32, HQ_ACT_SWIGLU_F32 = 0, 1, 2
HQ_FMT_E4M3, HQ_FMT_E2M1 = 0, 1
HQ_MAX_SECTIONS = 256
HQ_HOST_MAX_GROUPS = 32

EXPORTED = (
    "hq_version", "hq_status_string", "hq_group_rht_quant_workspace_size", "hq_workspace_init",
    "hq_get_error", "hq_group_rht_quant", "hq_group_rht_quant_sr", "hq_group_rht_quant_noalloc",
    "hq_group_rht_quant_host", "hq_group_rht_quant_host_device_bytes", "hq_cat_rotate_fp8",
    "hq_cat_rotate_fp8_workspace_size", "hq_cat_rotate_nvfp4", "hq_cat_rotate_nvfp4_workspace_size",
    "hq_swiglu_fp8_k128", "hq_swiglu_fp8_k128_workspace_size", "hq_convert", "hq_convert_e2m1_sr",
)


class HQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libhq.so (raises OSError if it is missing: build it first)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"{LIB_PATH} not found: run nvfp4_quantization_group_b200/_build.py")
        L = ctypes.CDLL(LIB_PATH)
        P, i64, sz, u = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_uint
        c_int = ctypes.c_int
        L.hq_version.restype = c_int
        L.hq_version.argtypes = []
        L.hq_status_string.restype = ctypes.c_char_p
        L.hq_status_string.argtypes = [c_int]
        L.hq_group_rht_quant_workspace_size.restype = sz
        L.hq_group_rht_quant_workspace_size.argtypes = [c_int]
        L.hq_workspace_init.restype = c_int
        L.hq_workspace_init.argtypes = [P, sz, P]
        L.hq_get_error.restype = c_int
        L.hq_get_error.argtypes = [P, sz, ctypes.POINTER(ctypes.c_uint32), P]
        L.hq_group_rht_quant.restype = c_int
        L.hq_group_rht_quant.argtypes = [P, i64, i64, P, c_int, ctypes.c_uint16, u,
                                         P, P, P, P, P, P, P, P, P, sz, P]
        L.hq_group_rht_quant_sr.restype = c_int
        L.hq_group_rht_quant_sr.argtypes = [P, i64, i64, P, c_int, ctypes.c_uint16, u, ctypes.c_uint64,
                                            ctypes.c_uint64, P, P, P, P, P, P, P, P, P, sz, P]
        L.hq_group_rht_quant_noalloc.restype = c_int
        L.hq_group_rht_quant_noalloc.argtypes = [P, i64, i64, P, c_int, ctypes.c_uint16, u,
                                                 P, P, P, P, P, P, P, P, P]
        L.hq_group_rht_quant_host_device_bytes.restype = sz
        L.hq_group_rht_quant_host_device_bytes.argtypes = [i64, i64, c_int]
        L.hq_group_rht_quant_host.restype = c_int
        L.hq_group_rht_quant_host.argtypes = [P, i64, i64, P, c_int, ctypes.c_uint16, u, ctypes.c_uint64,
                                              ctypes.c_uint64, P, P, P, P, P, P, P, P, P, sz, c_int, P, P, P]
        L.hq_cat_rotate_fp8.restype = c_int
        L.hq_cat_rotate_fp8.argtypes = [P, i64, c_int, P, i64, c_int, i64, c_int, c_int,
                                        P, P, c_int, i64, P, P, sz, P]
        L.hq_cat_rotate_fp8_workspace_size.restype = sz
        L.hq_cat_rotate_fp8_workspace_size.argtypes = []
        L.hq_cat_rotate_nvfp4.restype = c_int
        L.hq_cat_rotate_nvfp4.argtypes = [P, i64, c_int, P, i64, c_int, i64, c_int, c_int,
                                          P, P, P, c_int, i64, P, P, sz, P]
        L.hq_cat_rotate_nvfp4_workspace_size.restype = sz
        L.hq_cat_rotate_nvfp4_workspace_size.argtypes = []
        L.hq_swiglu_fp8_k128.restype = c_int
        L.hq_swiglu_fp8_k128.argtypes = [c_int, P, i64, i64, P, P, P, P, sz, P]
        L.hq_swiglu_fp8_k128_workspace_size.restype = sz
        L.hq_swiglu_fp8_k128_workspace_size.argtypes = []
        L.hq_convert.restype = c_int
        L.hq_convert.argtypes = [c_int, P, P, i64, P]
        L.hq_convert_e2m1_sr.restype = c_int
        L.hq_convert_e2m1_sr.argtypes = [P, P, P, i64, P]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().hq_status_string(int(status)).decode()


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _stream_or_null(stream):
    return None if stream is None else _stream(stream)


def _check(status: int, what: str) -> None:
    if status != HQ_OK:
        raise HQError(status, what)


# ------------------------------------------------------------- C ABI calls
def hq_version() -> int:
    return lib().hq_version()


def hq_group_rht_quant_workspace_size(num_sections: int) -> int:
    return int(lib().hq_group_rht_quant_workspace_size(int(num_sections)))


def hq_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check(lib().hq_workspace_init(_p(ws), ws.numel() * ws.element_size(), _stream(stream)), "hq_workspace_init")


def hq_get_error(ws: torch.Tensor, stream=None) -> int:
    err = ctypes.c_uint32(0)
    _check(lib().hq_get_error(_p(ws), ws.numel() * ws.element_size(), ctypes.byref(err), _stream(stream)),
           "hq_get_error")
    return int(err.value)


def hq_group_rht_quant(x, M, K, split_rows, S, sign_mask, flags, row_codes, row_sf, col_codes, col_sf,
                       amax_row, amax_col, sdec_row, sdec_col, ws, stream=None) -> None:
    splits = (ctypes.c_int64 * len(split_rows))(*[int(v) for v in split_rows])
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().hq_group_rht_quant(_p(x), int(M), int(K), ctypes.cast(splits, ctypes.c_void_p), int(S),
                                    int(sign_mask) & 0xFFFF, int(flags), _p(row_codes), _p(row_sf),
                                    _p(col_codes), _p(col_sf), _p(amax_row), _p(amax_col), _p(sdec_row),
                                    _p(sdec_col), _p(ws), ws_bytes, _stream(stream)), "hq_group_rht_quant")


def hq_group_rht_quant_sr(x, M, K, split_rows, S, sign_mask, flags, seed, offset, row_codes, row_sf, col_codes,
                          col_sf, amax_row, amax_col, sdec_row, sdec_col, ws, stream=None) -> None:
    splits = (ctypes.c_int64 * len(split_rows))(*[int(v) for v in split_rows])
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().hq_group_rht_quant_sr(_p(x), int(M), int(K), ctypes.cast(splits, ctypes.c_void_p), int(S),
                                       int(sign_mask) & 0xFFFF, int(flags), int(seed) & (2**64 - 1),
                                       int(offset) & (2**64 - 1), _p(row_codes), _p(row_sf), _p(col_codes),
                                       _p(col_sf), _p(amax_row), _p(amax_col), _p(sdec_row), _p(sdec_col), _p(ws),
                                       ws_bytes, _stream(stream)), "hq_group_rht_quant_sr")


def hq_group_rht_quant_noalloc(x, M, K, split_rows, S, sign_mask, flags, row_codes, row_sf, col_codes, col_sf,
                               amax_row, amax_col, sdec_row, sdec_col, stream=None) -> None:
    """hq_group_rht_quant with the library's fixed scratch array instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    splits = (ctypes.c_int64 * len(split_rows))(*[int(v) for v in split_rows])
    _check(lib().hq_group_rht_quant_noalloc(_p(x), int(M), int(K), ctypes.cast(splits, ctypes.c_void_p), int(S),
                                            int(sign_mask) & 0xFFFF, int(flags), _p(row_codes), _p(row_sf),
                                            _p(col_codes), _p(col_sf), _p(amax_row), _p(amax_col), _p(sdec_row),
                                            _p(sdec_col), _stream(stream)), "hq_group_rht_quant_noalloc")


def hq_group_rht_quant_host_device_bytes(M: int, K: int, S: int) -> int:
    return int(lib().hq_group_rht_quant_host_device_bytes(int(M), int(K), int(S)))


def hq_group_rht_quant_host(x, M, K, split_rows, S, sign_mask, flags, seed, offset, row_codes, row_sf, col_codes,
                            col_sf, amax_row, amax_col, sdec_row, sdec_col, dev_buf, groups=0, stream=None,
                            h2d_stream=None, d2h_stream=None) -> None:
    """x and the outputs are CPU tensors (page-locked for overlap); dev_buf a CUDA byte tensor of at least
    hq_group_rht_quant_host_device_bytes(M, K, S), zeroed once."""
    splits = (ctypes.c_int64 * len(split_rows))(*[int(v) for v in split_rows])
    _check(lib().hq_group_rht_quant_host(_p(x), int(M), int(K), ctypes.cast(splits, ctypes.c_void_p), int(S),
                                         int(sign_mask) & 0xFFFF, int(flags), int(seed) & (2**64 - 1),
                                         int(offset) & (2**64 - 1), _p(row_codes), _p(row_sf), _p(col_codes),
                                         _p(col_sf), _p(amax_row), _p(amax_col), _p(sdec_row), _p(sdec_col),
                                         _p(dev_buf), 0 if dev_buf is None else dev_buf.numel() * dev_buf.element_size(),
                                         int(groups), _stream(stream), _stream_or_null(h2d_stream),
                                         _stream_or_null(d2h_stream)), "hq_group_rht_quant_host")


def hq_cat_rotate_fp8(a, a_row_stride, a_width, b, b_row_stride, b_width, M, G, hadamard_n, out_fp8, scales,
                      scale_layout, scale_ld, amax_opt=None, stream=None) -> None:
    _check(lib().hq_cat_rotate_fp8(_p(a), int(a_row_stride), int(a_width), _p(b), int(b_row_stride),
                                   int(b_width), int(M), int(G), int(hadamard_n), _p(out_fp8), _p(scales),
                                   int(scale_layout), int(scale_ld), _p(amax_opt), None, 0, _stream(stream)),
           "hq_cat_rotate_fp8")


def hq_cat_rotate_fp8_workspace_size() -> int:
    return int(lib().hq_cat_rotate_fp8_workspace_size())


def hq_cat_rotate_nvfp4(a, a_row_stride, a_width, b, b_row_stride, b_width, M, G, hadamard_n, codes, block_sf, sdec,
                        scale_layout, scale_ld, amax_opt=None, stream=None) -> None:
    _check(lib().hq_cat_rotate_nvfp4(_p(a), int(a_row_stride), int(a_width), _p(b), int(b_row_stride),
                                     int(b_width), int(M), int(G), int(hadamard_n), _p(codes), _p(block_sf), _p(sdec),
                                     int(scale_layout), int(scale_ld), _p(amax_opt), None, 0, _stream(stream)),
           "hq_cat_rotate_nvfp4")


def hq_cat_rotate_nvfp4_workspace_size() -> int:
    return int(lib().hq_cat_rotate_nvfp4_workspace_size())


def hq_swiglu_fp8_k128(mode, inp, M, K_out, out_fp8, scales, amax_opt=None, stream=None) -> None:
    _check(lib().hq_swiglu_fp8_k128(int(mode), _p(inp), int(M), int(K_out), _p(out_fp8), _p(scales),
                                    _p(amax_opt), None, 0, _stream(stream)), "hq_swiglu_fp8_k128")


def hq_swiglu_fp8_k128_workspace_size() -> int:
    return int(lib().hq_swiglu_fp8_k128_workspace_size())


def hq_convert(fmt, inp, out, n, stream=None) -> None:
    _check(lib().hq_convert(int(fmt), _p(inp), _p(out), int(n), _stream(stream)), "hq_convert")


def hq_convert_e2m1_sr(inp, rnd, out, n, stream=None) -> None:
    _check(lib().hq_convert_e2m1_sr(_p(inp), _p(rnd), _p(out), int(n), _stream(stream)), "hq_convert_e2m1_sr")


# ------------------------------------------------- allocating conveniences
class HostStaging:
    """Device staging memory and the two copy streams of hq_group_rht_quant_host, for one shape; reusable."""

    def __init__(self, M: int, K: int, S: int, device="cuda"):
        nbytes = hq_group_rht_quant_host_device_bytes(M, K, S)
        if nbytes == 0:
            raise HQError(HQ_ERR_SHAPE, "HostStaging")
        self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=device)  # workspace rest state included
        self.h2d = torch.cuda.Stream(device=device)
        self.d2h = torch.cuda.Stream(device=device)


def host_outputs(M: int, K: int, S: int, flags: int = HQ_ROWWISE | HQ_COLWISE, pin: bool = True) -> dict:
    """Page-locked CPU output tensors for group_rht_quant_host (same names and shapes as group_outputs)."""
    out = {}
    u8 = dict(dtype=torch.uint8, pin_memory=pin)
    f32 = dict(dtype=torch.float32, pin_memory=pin)
    if flags & HQ_ROWWISE:
        out.update(row_codes=torch.empty((M, K // 2), **u8), row_sf=torch.empty((M, K // 16), **u8),
                   amax_row=torch.empty(S, **f32), sdec_row=torch.empty(S, **f32))
    if flags & HQ_COLWISE:
        out.update(col_codes=torch.empty(M * K // 2, **u8), col_sf=torch.empty(M * K // 16, **u8),
                   amax_col=torch.empty(S, **f32), sdec_col=torch.empty(S, **f32))
    return out


def group_rht_quant_host(x: torch.Tensor, split_rows, sign_mask: int, flags: int = HQ_ROWWISE | HQ_COLWISE,
                         staging: HostStaging | None = None, out: dict | None = None, groups: int = 0,
                         stream=None, seed: int | None = None, offset: int = 0) -> dict:
    """The grouped cast of a CPU BF16 [M, K] tensor into CPU outputs (hq_group_rht_quant_host): copies and
    casts overlap by section groups.  The outputs are complete once `stream` (default: the current one) is
    synchronized."""
    M, K = x.shape
    S = len(split_rows)
    if (flags & (HQ_ROW_SR | HQ_COL_SR)) and seed is None:
        raise HQError(HQ_ERR_UNSUPPORTED, "group_rht_quant_host: stochastic rounding needs a seed")
    if staging is None:
        staging = HostStaging(M, K, S)
    if out is None:
        out = host_outputs(M, K, S, flags)
    g = out.get
    hq_group_rht_quant_host(x, M, K, split_rows, S, sign_mask, flags, 0 if seed is None else seed, offset,
                            g("row_codes"), g("row_sf"), g("col_codes"), g("col_sf"), g("amax_row"),
                            g("amax_col"), g("sdec_row"), g("sdec_col"), staging.buf, groups, stream,
                            staging.h2d, staging.d2h)
    return out


def new_workspace(num_sections: int, device="cuda", stream=None) -> torch.Tensor:
    """A workspace for `num_sections` sections, put into its rest state once."""
    nbytes = hq_group_rht_quant_workspace_size(num_sections)
    if nbytes == 0:
        raise HQError(HQ_ERR_SHAPE, "new_workspace")
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    hq_workspace_init(ws, stream)
    return ws


def group_outputs(M: int, K: int, S: int, flags: int = HQ_ROWWISE | HQ_COLWISE, device="cuda") -> dict:
    u8 = dict(dtype=torch.uint8, device=device)
    f32 = dict(dtype=torch.float32, device=device)
    out = {}
    if flags & HQ_ROWWISE:
        out.update(row_codes=torch.empty((M, K // 2), **u8), row_sf=torch.empty((M, K // 16), **u8),
                   amax_row=torch.empty(S, **f32), sdec_row=torch.empty(S, **f32))
    if flags & HQ_COLWISE:
        out.update(col_codes=torch.empty(M * K // 2, **u8), col_sf=torch.empty(M * K // 16, **u8),
                   amax_col=torch.empty(S, **f32), sdec_col=torch.empty(S, **f32))
    return out


def group_rht_quant(x: torch.Tensor, split_rows, sign_mask: int, flags: int = HQ_ROWWISE | HQ_COLWISE,
                    ws: torch.Tensor | None = None, out: dict | None = None, stream=None, seed: int | None = None,
                    offset: int = 0) -> dict:
    """Grouped RHT16 + NVFP4 cast of a BF16 [M, K] CUDA tensor (see hq.h); with a seed, through
    hq_group_rht_quant_sr (stochastic rounding for HQ_ROW_SR / HQ_COL_SR)."""
    M, K = x.shape
    S = len(split_rows)
    if ws is None:
        ws = new_workspace(S, x.device, stream)
    if out is None:
        out = group_outputs(M, K, S, flags, x.device)
    g = out.get
    if seed is not None:
        hq_group_rht_quant_sr(x, M, K, split_rows, S, sign_mask, flags, seed, offset, g("row_codes"), g("row_sf"),
                              g("col_codes"), g("col_sf"), g("amax_row"), g("amax_col"), g("sdec_row"),
                              g("sdec_col"), ws, stream)
    else:
        hq_group_rht_quant(x, M, K, split_rows, S, sign_mask, flags, g("row_codes"), g("row_sf"), g("col_codes"),
                           g("col_sf"), g("amax_row"), g("amax_col"), g("sdec_row"), g("sdec_col"), ws, stream)
    return out


def cat_rotate_fp8(a: torch.Tensor, b: torch.Tensor | None, hadamard_n: int = 128,
                   scale_layout: int = HQ_SCALE_ROWMAJOR, scale_ld: int | None = None, want_amax: bool = False,
                   stream=None):
    """a: BF16 [M, G, a_width], b: BF16 [M, G, b_width] or None -> (codes [M, G*128], scales), and with
    want_amax a third item: the groups' amax in the scales' layout."""
    M, G, aw = a.shape
    bw = 0 if b is None else b.shape[-1]
    codes = torch.empty((M, G * 128), dtype=torch.uint8, device=a.device)
    if (scale_layout & ~HQ_FP8_UE8M0) == HQ_SCALE_ROWMAJOR:
        scales = torch.empty((M, G), dtype=torch.float32, device=a.device)
        ld = G
    else:
        ld = M if scale_ld is None else scale_ld
        scales = torch.empty((G, ld), dtype=torch.float32, device=a.device)
    amax = torch.empty_like(scales) if want_amax else None
    hq_cat_rotate_fp8(a, a.stride(0), aw, b, 0 if b is None else b.stride(0), bw, M, G, hadamard_n, codes,
                      scales, scale_layout, ld, amax, stream)
    return (codes, scales, amax) if want_amax else (codes, scales)


def cat_rotate_nvfp4(a: torch.Tensor, b: torch.Tensor | None, hadamard_n: int = 128,
                     scale_layout: int = HQ_SCALE_ROWMAJOR, scale_ld: int | None = None, want_amax: bool = False,
                     stream=None) -> dict:
    """a: BF16 [M, G, a_width], b: BF16 [M, G, b_width] or None -> dict with codes [M, G*64],
    block_sf [M, G*8], sdec (per vector, the scales' layout) and, with want_amax, amax."""
    M, G, aw = a.shape
    bw = 0 if b is None else b.shape[-1]
    dev = a.device
    out = {"codes": torch.empty((M, G * 64), dtype=torch.uint8, device=dev),
           "block_sf": torch.empty((M, G * 8), dtype=torch.uint8, device=dev)}
    if (scale_layout & ~HQ_SF_SWIZZLED) == HQ_SCALE_ROWMAJOR:
        out["sdec"] = torch.empty((M, G), dtype=torch.float32, device=dev)
        ld = G
    else:
        ld = M if scale_ld is None else scale_ld
        out["sdec"] = torch.empty((G, ld), dtype=torch.float32, device=dev)
    if want_amax:
        out["amax"] = torch.empty_like(out["sdec"])
    hq_cat_rotate_nvfp4(a, a.stride(0), aw, b, 0 if b is None else b.stride(0), bw, M, G, hadamard_n, out["codes"],
                        out["block_sf"], out["sdec"], scale_layout, ld, out.get("amax"), stream)
    return out


def swiglu_fp8_k128(mode: int, inp: torch.Tensor, K_out: int, want_amax: bool = False, stream=None):
    """K128 FP8 quantization (modes HQ_ACT_*) -> (codes [M, K_out], scales [M, K_out/128]), and with
    want_amax a third item: the groups' amax [M, K_out/128]."""
    M = inp.shape[0]
    codes = torch.empty((M, K_out), dtype=torch.uint8, device=inp.device)
    scales = torch.empty((M, K_out // 128), dtype=torch.float32, device=inp.device)
    amax = torch.empty_like(scales) if want_amax else None
    hq_swiglu_fp8_k128(mode, inp, M, K_out, codes, scales, amax, stream)
    return (codes, scales, amax) if want_amax else (codes, scales)
