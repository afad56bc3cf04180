"""Python binding of libfp8q.so (the C ABI declared in include/fp8q.h).

Argument marshalling only: every step of quantization and GEMM runs in the library's CUDA
kernels.  PyTorch supplies device memory (outputs are allocated with torch) and the current
CUDA stream.  There is no CPU fallback: if the library is missing or no CUDA device is
present, the calls raise.

Two layers, same names as the C ABI:
  * ``fp8q_quantize_1x128(...)`` etc. take raw integers/pointers exactly like the C calls;
  * ``quantize_1x128(x, ...)``, ``quantize_128x128``, ``quantize_mx32``, ``quantize_tensor``,
    ``rht16_quantize_sr``, ``gemm`` take torch tensors, allocate the outputs and call them.
"""
import ctypes
import os

import torch

__all__ = [
    "FP8Q_OK", "FP8Q_BLOCKWISE", "FP8Q_MXFP8", "FP8Q_PERTENSOR", "FP8Q_NVFP4",
    "FP8Q_FPROP", "FP8Q_DGRAD", "FP8Q_WGRAD", "FP8Q_SF_ROWMAJOR", "FP8Q_SF_MMA_TILED",
    "FP4Q_ROW", "FP4Q_COL", "Fp8qError", "lib", "library_path",
    "fp8q_quantize_1x128", "fp8q_quantize_128x128", "fp8q_quantize_mx32", "fp8q_quantize_tensor",
    "fp8q_quantize_tensor_noalloc", "fp8q_quantize_128x128_grouped", "fp8q_quantize_tensor_delayed",
    "fp4q_rht16_quantize_sr", "fp4q_quantize_2d16", "FP8Q_E4M3", "FP8Q_E5M2", "fp8q_gemm_blockscaled", "fp8q_sf_bytes",
    "fp8q_get_device_status", "fp8q_selftest_bounded_wait", "fp8q_status_string", "fp8q_version", "GemmArgs",
    "quantize_1x128", "quantize_128x128", "quantize_128x128_grouped", "quantize_tensor_delayed", "quantize_mx32", "quantize_tensor", "rht16_quantize_sr",
    "quantize_nvfp4_2d16", "gemm", "gemm_workspace_bytes", "device_status", "EXPORTED_SYMBOLS",
    "fp8q_quantize_multi", "fp8q_gemm_workspace_bytes", "QuantItem", "FP8Q_ITEM_1X128", "FP8Q_ITEM_128X128", "FP8Q_MAX_QUANT_ITEMS",
    "quantize_multi",
]

FP8Q_OK = 0
FP8Q_ERR_NULL, FP8Q_ERR_SHAPE, FP8Q_ERR_ALIGN, FP8Q_ERR_UNSUPPORTED, FP8Q_ERR_CUDA, FP8Q_ERR_TIMEOUT = 1, 2, 3, 4, 5, 6
FP8Q_ERR_DEVICE_ARG = 7
FP8Q_BLOCKWISE, FP8Q_MXFP8, FP8Q_PERTENSOR, FP8Q_NVFP4 = 0, 1, 2, 3
FP8Q_FPROP, FP8Q_DGRAD, FP8Q_WGRAD = 0, 1, 2
FP8Q_SF_ROWMAJOR, FP8Q_SF_MMA_TILED = 0, 1
FP4Q_ROW, FP4Q_COL = 1, 2
FP8Q_E4M3, FP8Q_E5M2 = 0, 1
FP8Q_ITEM_1X128, FP8Q_ITEM_128X128 = 0, 1
FP8Q_MAX_QUANT_ITEMS = 8

EXPORTED_SYMBOLS = [
    "fp8q_quantize_1x128", "fp8q_quantize_128x128", "fp8q_quantize_mx32", "fp8q_quantize_tensor",
    "fp4q_rht16_quantize_sr", "fp8q_gemm_blockscaled", "fp8q_sf_bytes", "fp8q_get_device_status",
    "fp8q_release_scratch", "fp8q_status_string", "fp8q_version", "fp8q_quantize_tensor_noalloc",
    "fp8q_selftest_bounded_wait", "fp8q_quantize_128x128_grouped", "fp8q_quantize_tensor_delayed",
    "fp4q_quantize_2d16", "fp8q_quantize_multi", "fp8q_gemm_workspace_bytes",
]

library_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfp8q.so")


class Fp8qError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: status {status} ({_status_str(status)})")


class QuantItem(ctypes.Structure):
    """Mirror of fp8q_quant_item (field order and types as in include/fp8q.h)."""
    _fields_ = [
        ("kind", ctypes.c_int32), ("x", ctypes.c_void_p),
        ("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("ld_x", ctypes.c_int64),
        ("q_row", ctypes.c_void_p), ("s_row", ctypes.c_void_p), ("ld_s_row", ctypes.c_int64),
        ("q_col", ctypes.c_void_p), ("s_col", ctypes.c_void_p), ("ld_s_col", ctypes.c_int64),
        ("q_t", ctypes.c_void_p), ("q", ctypes.c_void_p), ("s", ctypes.c_void_p),
    ]


class GemmArgs(ctypes.Structure):
    """Mirror of fp8q_gemm_args (field order and types as in include/fp8q.h)."""
    _fields_ = [
        ("recipe", ctypes.c_int), ("layout", ctypes.c_int),
        ("M", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
        ("a", ctypes.c_void_p), ("a_scale", ctypes.c_void_p), ("lda", ctypes.c_int64), ("ld_sa", ctypes.c_int64),
        ("b", ctypes.c_void_p), ("b_scale", ctypes.c_void_p), ("ldb", ctypes.c_int64), ("ld_sb", ctypes.c_int64),
        ("a_global", ctypes.c_void_p), ("b_global", ctypes.c_void_p),
        ("c", ctypes.c_void_p), ("ldc", ctypes.c_int64),
        ("m_offsets", ctypes.c_void_p), ("num_groups", ctypes.c_int32),
        ("c_fp32_accumulate", ctypes.c_int32),
        ("a_format", ctypes.c_int32), ("b_format", ctypes.c_int32),
        ("q_out", ctypes.c_void_p), ("s_out", ctypes.c_void_p),
        ("ld_q_out", ctypes.c_int64), ("ld_s_out", ctypes.c_int64),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_int64),
    ]


_LIB = None
_i64, _u64, _vp, _int = ctypes.c_int64, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_int


def lib():
    """Loads libfp8q.so once; raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(library_path):
            raise ImportError(f"{library_path} is missing: build it with "
                              "`python -m fp4_precision_gemm_b200.build`")
        L = ctypes.CDLL(library_path)
        L.fp8q_quantize_1x128.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _i64, _vp]
        L.fp8q_quantize_128x128.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp]
        L.fp8q_quantize_128x128_grouped.argtypes = [_vp, _i64, _i64, _i64, _i64, _vp, _vp, _vp, _vp]
        L.fp8q_quantize_mx32.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _int, _vp]
        L.fp8q_quantize_tensor.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp, _vp]
        L.fp8q_quantize_tensor_noalloc.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp, _vp]
        L.fp8q_quantize_tensor_delayed.argtypes = [_vp, _i64, _i64, _i64, _vp, ctypes.c_int32, ctypes.c_int32, _int,
                                                   _vp, _vp, _vp]
        L.fp4q_rht16_quantize_sr.argtypes = [_vp, _i64, _i64, _i64, _int, _u64, _int, _u64,
                                             _vp, _vp, _vp, _vp, _vp, _vp, _int, _vp]
        L.fp4q_quantize_2d16.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _int, _vp]
        L.fp8q_gemm_blockscaled.argtypes = [ctypes.POINTER(GemmArgs), _vp]
        L.fp8q_gemm_workspace_bytes.argtypes = [ctypes.POINTER(GemmArgs)]
        L.fp8q_gemm_workspace_bytes.restype = ctypes.c_size_t
        L.fp8q_quantize_multi.argtypes = [ctypes.POINTER(QuantItem), ctypes.c_int32, _vp]
        L.fp8q_sf_bytes.argtypes = [_int, _i64, _i64, _int]
        L.fp8q_sf_bytes.restype = ctypes.c_size_t
        L.fp8q_get_device_status.argtypes = [_vp]
        L.fp8q_selftest_bounded_wait.argtypes = [_u64, _vp]
        L.fp8q_release_scratch.argtypes = []
        L.fp8q_status_string.argtypes = [_int]
        L.fp8q_status_string.restype = ctypes.c_char_p
        L.fp8q_version.argtypes = []
        L.fp8q_version.restype = ctypes.c_char_p
        for name in EXPORTED_SYMBOLS:
            f = getattr(L, name)
            if f.restype is ctypes.c_int or name in ("fp8q_quantize_1x128", "fp8q_quantize_128x128",
                                                     "fp8q_quantize_mx32", "fp8q_quantize_tensor",
                                                     "fp4q_rht16_quantize_sr", "fp8q_gemm_blockscaled",
                                                     "fp8q_get_device_status", "fp8q_release_scratch",
                                                     "fp8q_selftest_bounded_wait", "fp8q_quantize_128x128_grouped",
                                                     "fp8q_quantize_tensor_delayed", "fp4q_quantize_2d16",
                                                     "fp8q_quantize_multi"):
                f.restype = ctypes.c_int
        _LIB = L
    return _LIB


def _status_str(st):
    try:
        return lib().fp8q_status_string(st).decode()
    except Exception:  # noqa: BLE001 - message only
        return "?"


def _check(st, where):
    if st != FP8Q_OK:
        raise Fp8qError(st, where)


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


# --------------------------------------------------------------------------- raw C calls
def fp8q_quantize_1x128(x, rows, cols, ld_x, q_row, s_row, ld_s_row, q_col, s_col, ld_s_col, stream):
    return lib().fp8q_quantize_1x128(x, rows, cols, ld_x, q_row, s_row, ld_s_row, q_col, s_col, ld_s_col, stream)


def fp8q_quantize_128x128(w, K, N, ld_w, q_t, q, s, stream):
    return lib().fp8q_quantize_128x128(w, K, N, ld_w, q_t, q, s, stream)


def fp8q_quantize_multi(items, n_items, stream):
    """items: a ctypes array of QuantItem (or None with n_items == 0)."""
    return lib().fp8q_quantize_multi(items, n_items, stream)


def fp8q_quantize_128x128_grouped(w, groups, K, N, ld_w, q_t, q, s, stream):
    return lib().fp8q_quantize_128x128_grouped(w, groups, K, N, ld_w, q_t, q, s, stream)


def fp8q_quantize_mx32(x, rows, cols, ld_x, q_row, e_row, q_col, e_col, sf_layout, stream):
    return lib().fp8q_quantize_mx32(x, rows, cols, ld_x, q_row, e_row, q_col, e_col, sf_layout, stream)


def fp8q_quantize_tensor(x, rows, cols, ld_x, q, s_dec, stream):
    return lib().fp8q_quantize_tensor(x, rows, cols, ld_x, q, s_dec, stream)


def fp8q_quantize_tensor_delayed(x, rows, cols, ld_x, hist, hlen, hpos, fmt, q, s_dec, stream):
    return lib().fp8q_quantize_tensor_delayed(x, rows, cols, ld_x, hist, hlen, hpos, fmt, q, s_dec, stream)


def fp8q_quantize_tensor_noalloc(x, rows, cols, ld_x, q, s_dec, stream):
    """Per-tensor quantization that allocates no device memory (scratch in the library's
    fixed device array); for callers that cannot let a library allocate."""
    return lib().fp8q_quantize_tensor_noalloc(x, rows, cols, ld_x, q, s_dec, stream)


def fp4q_rht16_quantize_sr(x, rows, cols, ld_x, rht, rht_seed, sr, sr_seed, q_row, sf_row, g_row,
                           q_col, sf_col, g_col, sf_layout, stream):
    return lib().fp4q_rht16_quantize_sr(x, rows, cols, ld_x, rht, rht_seed, sr, sr_seed, q_row, sf_row, g_row,
                                        q_col, sf_col, g_col, sf_layout, stream)


def fp4q_quantize_2d16(x, rows, cols, ld_x, q_row, sf_row, q_col, sf_col, g_dec, sf_layout, stream):
    return lib().fp4q_quantize_2d16(x, rows, cols, ld_x, q_row, sf_row, q_col, sf_col, g_dec, sf_layout, stream)


def fp8q_gemm_blockscaled(args, stream):
    return lib().fp8q_gemm_blockscaled(ctypes.byref(args), stream)


def fp8q_gemm_workspace_bytes(args):
    return lib().fp8q_gemm_workspace_bytes(ctypes.byref(args))


def fp8q_sf_bytes(recipe, outer, inner, layout):
    return int(lib().fp8q_sf_bytes(recipe, outer, inner, layout))


def fp8q_get_device_status(stream):
    return lib().fp8q_get_device_status(stream)


def fp8q_selftest_bounded_wait(limit_ns, stream):
    return lib().fp8q_selftest_bounded_wait(limit_ns, stream)


def fp8q_status_string(st):
    return lib().fp8q_status_string(st).decode()


def fp8q_version():
    return lib().fp8q_version().decode()


# --------------------------------------------------------------------------- tensor API
def _check_bf16(x, name="x"):
    if not (x.is_cuda and x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1):
        raise ValueError(f"{name} must be a 2-D row-major CUDA bf16 tensor")


def quantize_1x128(x, rowwise=True, colwise=False, stream=None):
    """1x128 tiles.  Returns dict with q_row (R, C) uint8, s_row (C/128, R) float32 and/or
    q_col (C, R) uint8, s_col (R/128, C) float32."""
    _check_bf16(x)
    R, C = x.shape
    out = {}
    dev = x.device
    if rowwise:
        out["q_row"] = torch.empty((R, C), dtype=torch.uint8, device=dev)
        out["s_row"] = torch.empty((C // 128, max(R, 1) + (-max(R, 1)) % 4), dtype=torch.float32, device=dev)
    if colwise:
        out["q_col"] = torch.empty((C, R), dtype=torch.uint8, device=dev)
        out["s_col"] = torch.empty((R // 128, C + (-C) % 4), dtype=torch.float32, device=dev)
    st = fp8q_quantize_1x128(_ptr(x), R, C, x.stride(0), _ptr(out.get("q_row")), _ptr(out.get("s_row")),
                             out["s_row"].shape[1] if rowwise else 0, _ptr(out.get("q_col")),
                             _ptr(out.get("s_col")), out["s_col"].shape[1] if colwise else 0, _stream(stream))
    _check(st, "fp8q_quantize_1x128")
    return out


def quantize_128x128(w, transposed=True, plain=True, stream=None):
    """128x128 blocks of W (K x N).  Returns q_t (N, K), q (K, N), s (N/128, K/128)."""
    _check_bf16(w, "w")
    K, N = w.shape
    dev = w.device
    out = {"s": torch.empty((N // 128, K // 128), dtype=torch.float32, device=dev)}
    if transposed:
        out["q_t"] = torch.empty((N, K), dtype=torch.uint8, device=dev)
    if plain:
        out["q"] = torch.empty((K, N), dtype=torch.uint8, device=dev)
    st = fp8q_quantize_128x128(_ptr(w), K, N, w.stride(0), _ptr(out.get("q_t")), _ptr(out.get("q")),
                               _ptr(out["s"]), _stream(stream))
    _check(st, "fp8q_quantize_128x128")
    return out


def quantize_multi(specs, stream=None):
    """Several quantizations in one launch.  specs: a list of ("1x128", x, rowwise, colwise)
    and ("128x128", w, transposed, plain) tuples.  Returns one output dict per spec, laid
    out exactly as quantize_1x128 / quantize_128x128 return them."""
    items = (QuantItem * max(len(specs), 1))()
    outs = []
    n = 0
    for spec in specs:
        kind, x, a, b = spec
        _check_bf16(x)
        R, C = x.shape
        dev = x.device
        it = items[n] if x.numel() else QuantItem()   # an empty tensor has nothing to launch
        n += 1 if x.numel() else 0
        it.x, it.rows, it.cols, it.ld_x = x.data_ptr(), R, C, x.stride(0)
        out = {}
        if kind == "1x128":
            it.kind = FP8Q_ITEM_1X128
            if a:
                out["q_row"] = torch.empty((R, C), dtype=torch.uint8, device=dev)
                out["s_row"] = torch.empty((C // 128, max(R, 1) + (-max(R, 1)) % 4), dtype=torch.float32, device=dev)
                it.q_row, it.s_row, it.ld_s_row = out["q_row"].data_ptr(), out["s_row"].data_ptr(), out["s_row"].shape[1]
            if b:
                out["q_col"] = torch.empty((C, R), dtype=torch.uint8, device=dev)
                out["s_col"] = torch.empty((R // 128, C + (-C) % 4), dtype=torch.float32, device=dev)
                it.q_col, it.s_col, it.ld_s_col = out["q_col"].data_ptr(), out["s_col"].data_ptr(), out["s_col"].shape[1]
        elif kind == "128x128":
            it.kind = FP8Q_ITEM_128X128
            out["s"] = torch.empty((C // 128, R // 128), dtype=torch.float32, device=dev)
            it.s = out["s"].data_ptr()
            if a:
                out["q_t"] = torch.empty((C, R), dtype=torch.uint8, device=dev)
                it.q_t = out["q_t"].data_ptr()
            if b:
                out["q"] = torch.empty((R, C), dtype=torch.uint8, device=dev)
                it.q = out["q"].data_ptr()
        else:
            raise ValueError(f"unknown quantization kind {kind!r}")
        outs.append(out)
    st = fp8q_quantize_multi(items, n, _stream(stream))
    _check(st, "fp8q_quantize_multi")
    return outs


def quantize_128x128_grouped(w, transposed=True, plain=True, stream=None):
    """128x128 blocks of every matrix of a stack W (G x K x N, contiguous matrices) in one
    call.  Returns q_t (G, N, K), q (G, K, N), s (G, N/128, K/128)."""
    if w.dim() != 3 or w.dtype != torch.bfloat16 or not w.is_cuda:
        raise ValueError("w must be a CUDA bfloat16 tensor of shape (G, K, N)")
    if w.stride(2) != 1 or w.stride(0) != w.shape[1] * w.stride(1):
        raise ValueError("w must hold contiguous row-major matrices (row stride may be padded)")
    G, K, N = w.shape
    dev = w.device
    out = {"s": torch.empty((G, N // 128, K // 128), dtype=torch.float32, device=dev)}
    if transposed:
        out["q_t"] = torch.empty((G, N, K), dtype=torch.uint8, device=dev)
    if plain:
        out["q"] = torch.empty((G, K, N), dtype=torch.uint8, device=dev)
    st = fp8q_quantize_128x128_grouped(_ptr(w), G, K, N, w.stride(1), _ptr(out.get("q_t")), _ptr(out.get("q")),
                                       _ptr(out["s"]), _stream(stream))
    _check(st, "fp8q_quantize_128x128_grouped")
    return out


def quantize_mx32(x, rowwise=True, colwise=False, sf_layout=FP8Q_SF_ROWMAJOR, stream=None):
    """MXFP8.  Returns q_row (R, C) + e8m0_row, and/or q_col (C, R) + e8m0_col (flat uint8
    buffers sized by fp8q_sf_bytes for the chosen layout)."""
    _check_bf16(x)
    R, C = x.shape
    dev = x.device
    out = {}
    if rowwise:
        out["q_row"] = torch.empty((R, C), dtype=torch.uint8, device=dev)
        out["e8m0_row"] = torch.empty(fp8q_sf_bytes(FP8Q_MXFP8, R, C, sf_layout), dtype=torch.uint8, device=dev)
    if colwise:
        out["q_col"] = torch.empty((C, R), dtype=torch.uint8, device=dev)
        out["e8m0_col"] = torch.empty(fp8q_sf_bytes(FP8Q_MXFP8, C, R, sf_layout), dtype=torch.uint8, device=dev)
    st = fp8q_quantize_mx32(_ptr(x), R, C, x.stride(0), _ptr(out.get("q_row")), _ptr(out.get("e8m0_row")),
                            _ptr(out.get("q_col")), _ptr(out.get("e8m0_col")), sf_layout, _stream(stream))
    _check(st, "fp8q_quantize_mx32")
    return out


def quantize_tensor(x, stream=None):
    """Per-tensor current scaling.  Returns q (R, C) uint8 and s_dec (1,) float32."""
    _check_bf16(x)
    R, C = x.shape
    out = {"q": torch.empty((R, C), dtype=torch.uint8, device=x.device),
           "s_dec": torch.empty((1,), dtype=torch.float32, device=x.device)}
    st = fp8q_quantize_tensor(_ptr(x), R, C, x.stride(0), _ptr(out["q"]), _ptr(out["s_dec"]), _stream(stream))
    _check(st, "fp8q_quantize_tensor")
    return out


def quantize_tensor_delayed(x, amax_history, history_pos, fmt=FP8Q_E4M3, stream=None):
    """Per-tensor delayed scaling: scale from max(amax_history) (float32 CUDA tensor, updated
    in place at history_pos with this tensor's amax).  Returns q (R, C) uint8, s_dec (1,)."""
    _check_bf16(x)
    if not (amax_history.is_cuda and amax_history.dtype == torch.float32 and amax_history.dim() == 1):
        raise ValueError("amax_history must be a 1-D float32 CUDA tensor")
    R, C = x.shape
    out = {"q": torch.empty((R, C), dtype=torch.uint8, device=x.device),
           "s_dec": torch.empty((1,), dtype=torch.float32, device=x.device)}
    st = fp8q_quantize_tensor_delayed(_ptr(x), R, C, x.stride(0), _ptr(amax_history), amax_history.numel(),
                                      history_pos, fmt, _ptr(out["q"]), _ptr(out["s_dec"]), _stream(stream))
    _check(st, "fp8q_quantize_tensor_delayed")
    return out


def rht16_quantize_sr(x, rowwise=True, colwise=False, rht=0, rht_seed=0, sr=0, sr_seed=0,
                      sf_layout=FP8Q_SF_ROWMAJOR, stream=None):
    """NVFP4.  rht / sr are FP4Q_ROW | FP4Q_COL masks.  Returns q_row (R, C/2), sf_row,
    g_row (1,) and/or q_col (C, R/2), sf_col, g_col (1,)."""
    _check_bf16(x)
    R, C = x.shape
    dev = x.device
    out = {}
    if rowwise:
        out["q_row"] = torch.empty((R, C // 2), dtype=torch.uint8, device=dev)
        out["sf_row"] = torch.empty(fp8q_sf_bytes(FP8Q_NVFP4, R, C, sf_layout), dtype=torch.uint8, device=dev)
        out["g_row"] = torch.empty((1,), dtype=torch.float32, device=dev)
    if colwise:
        out["q_col"] = torch.empty((C, R // 2), dtype=torch.uint8, device=dev)
        out["sf_col"] = torch.empty(fp8q_sf_bytes(FP8Q_NVFP4, C, R, sf_layout), dtype=torch.uint8, device=dev)
        out["g_col"] = torch.empty((1,), dtype=torch.float32, device=dev)
    st = fp4q_rht16_quantize_sr(_ptr(x), R, C, x.stride(0), rht, rht_seed, sr, sr_seed,
                                _ptr(out.get("q_row")), _ptr(out.get("sf_row")), _ptr(out.get("g_row")),
                                _ptr(out.get("q_col")), _ptr(out.get("sf_col")), _ptr(out.get("g_col")),
                                sf_layout, _stream(stream))
    _check(st, "fp4q_rht16_quantize_sr")
    return out


def quantize_nvfp4_2d16(w, rowwise=True, colwise=True, sf_layout=FP8Q_SF_MMA_TILED, stream=None):
    """NVFP4 weights with one scale per 16x16 block.  Returns q_row (R, C/2), sf_row and/or
    q_col (C, R/2), sf_col, and g (1,), the decode scale both layouts share."""
    _check_bf16(w, "w")
    R, C = w.shape
    dev = w.device
    out = {"g": torch.empty((1,), dtype=torch.float32, device=dev)}
    if rowwise:
        out["q_row"] = torch.empty((R, C // 2), dtype=torch.uint8, device=dev)
        out["sf_row"] = torch.empty(fp8q_sf_bytes(FP8Q_NVFP4, R, C, sf_layout), dtype=torch.uint8, device=dev)
    if colwise:
        out["q_col"] = torch.empty((C, R // 2), dtype=torch.uint8, device=dev)
        out["sf_col"] = torch.empty(fp8q_sf_bytes(FP8Q_NVFP4, C, R, sf_layout), dtype=torch.uint8, device=dev)
    st = fp4q_quantize_2d16(_ptr(w), R, C, w.stride(0), _ptr(out.get("q_row")), _ptr(out.get("sf_row")),
                            _ptr(out.get("q_col")), _ptr(out.get("sf_col")), _ptr(out["g"]), sf_layout,
                            _stream(stream))
    _check(st, "fp4q_quantize_2d16")
    return out


def _gemm_args(a, b, recipe, layout, a_scale, b_scale, ld_sa, ld_sb, a_global, b_global, K, m_offsets, out,
               accumulate_fp32, a_format, b_format, q_out, s_out):
    """The C ABI's argument block for gemm() (and the output tensor it writes)."""
    M = a.shape[0]
    grouped = m_offsets is not None
    N = b.shape[1] if grouped else b.shape[0]
    if K is None:
        K = a.shape[1] * (2 if recipe == FP8Q_NVFP4 else 1)
    if accumulate_fp32 and (out is None or out.dtype != torch.float32):
        raise ValueError("accumulate_fp32 needs an FP32 `out` tensor to update")
    c = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    args = GemmArgs()
    args.recipe, args.layout = recipe, layout
    args.M, args.N, args.K = M, N, K
    args.a, args.lda = a.data_ptr(), a.stride(0)
    args.b, args.ldb = b.data_ptr(), b.stride(-2)
    args.a_scale = a_scale.data_ptr() if a_scale is not None else None
    args.b_scale = b_scale.data_ptr() if b_scale is not None else None
    args.ld_sa = ld_sa if ld_sa is not None else (a_scale.shape[-1] if (a_scale is not None and a_scale.dim() == 2) else 0)
    args.ld_sb = ld_sb if ld_sb is not None else (b_scale.shape[-1] if (b_scale is not None and b_scale.dim() >= 2) else 0)
    args.a_global = a_global.data_ptr() if a_global is not None else None
    args.b_global = b_global.data_ptr() if b_global is not None else None
    args.c, args.ldc = c.data_ptr(), c.stride(0)
    args.m_offsets = m_offsets.data_ptr() if grouped else None
    args.num_groups = (m_offsets.numel() - 1) if grouped else 0
    args.c_fp32_accumulate = 1 if accumulate_fp32 else 0
    args.a_format, args.b_format = a_format, b_format
    if q_out is not None or s_out is not None:
        args.q_out = q_out.data_ptr() if q_out is not None else None
        args.s_out = s_out.data_ptr() if s_out is not None else None
        args.ld_q_out = q_out.stride(0) if q_out is not None else 0
        args.ld_s_out = s_out.stride(0) if s_out is not None else 0
    return args, c


def gemm(a, b, recipe=FP8Q_BLOCKWISE, layout=FP8Q_FPROP, a_scale=None, b_scale=None, ld_sa=None, ld_sb=None,
         a_global=None, b_global=None, K=None, m_offsets=None, out=None, accumulate_fp32=False,
         a_format=0, b_format=0, q_out=None, s_out=None, stream=None, split_tail=True):
    """C = A . B^T (BF16).  a: (M, K or K/2) uint8 codes, b: (N, ...) or (G, N, ...) uint8.
    Scales as the C ABI describes for the recipe.  Returns C (M, N) bf16.
    accumulate_fp32 (BLOCKWISE): `out` is an FP32 (M, N) tensor updated in place, C += A . B^T.
    q_out (M, N) uint8 and s_out (N/128, M) float32 (BLOCKWISE): also receive the 1x128
    rowwise quantization of the BF16 C, made in the GEMM's epilogue.
    split_tail (BLOCKWISE, not grouped, no q_out): give the call the workspace it asks for
    (fp8q_gemm_workspace_bytes), taken from torch's caching allocator on the call's stream, so
    that a mostly idle last wave is split into K ranges."""
    args, c = _gemm_args(a, b, recipe, layout, a_scale, b_scale, ld_sa, ld_sb, a_global, b_global, K, m_offsets,
                         out, accumulate_fp32, a_format, b_format, q_out, s_out)
    ws = None
    if split_tail and recipe == FP8Q_BLOCKWISE:
        nbytes = fp8q_gemm_workspace_bytes(args)
        if nbytes > 0:
            ws = torch.empty(nbytes, dtype=torch.uint8, device=a.device)
            if stream is not None:
                ws.record_stream(stream)
            args.workspace, args.workspace_bytes = ws.data_ptr(), nbytes
    _check(fp8q_gemm_blockscaled(args, _stream(stream)), "fp8q_gemm_blockscaled")
    return c


def gemm_workspace_bytes(M, N, K, recipe=FP8Q_BLOCKWISE, layout=FP8Q_FPROP, accumulate_fp32=False,
                         fused_quant=False, grouped=False):
    """Workspace bytes gemm() gives a call of this kind and size (0: the call launches one
    kernel; otherwise two: the tiles with the last wave's K ranges, then the sum of the ranges)."""
    args = GemmArgs()
    args.recipe, args.layout = recipe, layout
    args.M, args.N, args.K = M, N, K
    args.c_fp32_accumulate = 1 if accumulate_fp32 else 0
    args.num_groups = 1 if grouped else 0
    if fused_quant:
        args.q_out, args.s_out = 16, 16          # only their presence is read
    return fp8q_gemm_workspace_bytes(args)


def device_status(stream=None):
    """Synchronizes the stream; returns and clears the device status word."""
    return fp8q_get_device_status(_stream(stream))
