"""Python binding of the MLA decode C ABI (``libmla_b200.so``, declared in ``include/mla.h``).

Argument marshalling only: every function takes torch tensors already on the GPU, checks dtype,
shape and contiguity, and passes raw device pointers plus the current CUDA stream to the
library.  Every step of the computation runs in the library's kernels; there is no fallback.
Functions keep the C names: ``mla_cache_append``, ``mla_absorb_q``, ``mla_decode_attn``,
``mla_out_proj``, plus ``mla_workspace_size``, ``mla_cache_row_bytes``, ``mla_get_status``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla_b200.so")

MLA_BF16 = 0
MLA_FP32 = 1

STATUS_BAD_PAGE = 0x1
STATUS_BAD_LENGTH = 0x2
STATUS_TIMEOUT = 0x4
STATUS_BAD_POSITION = 0x8

ERRORS = {
    -1: "MLA_ERR_NULL_ARG", -2: "MLA_ERR_DIMS", -3: "MLA_ERR_ALIGN", -4: "MLA_ERR_WORKSPACE",
    -5: "MLA_ERR_ARG", -6: "MLA_ERR_CUDA", -7: "MLA_ERR_DEVICE",
}


class MlaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        detail = _error_detail() if code == -6 else ""
        super().__init__(f"{where}: {ERRORS.get(code, code)} ({_error_string(code)})"
                         + (f": {detail}" if detail else ""))


class mla_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("d_c", ctypes.c_int32),
                ("d_rope", ctypes.c_int32), ("d_nope", ctypes.c_int32), ("d_v", ctypes.c_int32),
                ("d_model", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("rope_theta", ctypes.c_float)]


def dims(batch: int, n_heads: int = 128, d_model: int = 7168, dtype=torch.bfloat16,
         rope_theta: float = 10000.0) -> mla_dims:
    return mla_dims(batch, n_heads, 512, 64, 128, 128, d_model, 64,
                    MLA_BF16 if dtype == torch.bfloat16 else MLA_FP32, rope_theta)


class mla_layer(ctypes.Structure):
    _fields_ = [("w_dkv", ctypes.c_void_p), ("w_kr", ctypes.c_void_p), ("w_q", ctypes.c_void_p),
                ("w_uk", ctypes.c_void_p), ("w_uv", ctypes.c_void_p), ("w_o", ctypes.c_void_p),
                ("cache_pool", ctypes.c_void_p), ("num_pages", ctypes.c_int32),
                ("page_table", ctypes.c_void_p), ("max_pages", ctypes.c_int32),
                ("w_dkv_scale", ctypes.c_void_p), ("w_kr_scale", ctypes.c_void_p),
                ("w_q_scale", ctypes.c_void_p), ("w_o_scale", ctypes.c_void_p)]


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int32
_SZ = ctypes.c_size_t
_SIGS = {
    "mla_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(mla_dims), _I]),
    "mla_cache_row_bytes": (ctypes.c_int64, [ctypes.POINTER(mla_dims)]),
    "mla_cache_append": (ctypes.c_int, [ctypes.POINTER(mla_dims), _P, _P, _P, _P, _P, _I, _P, _I,
                                        _P, _SZ, _P]),
    "mla_absorb_q": (ctypes.c_int, [ctypes.POINTER(mla_dims), _P, _P, _P, _P, _P, _P, _P, _SZ,
                                    _P]),
    "mla_append_absorb": (ctypes.c_int, [ctypes.POINTER(mla_dims), _P, _P, _P, _P, _P, _P, _P,
                                         _I, _P, _I, _P, _P, _P, _SZ, _P]),
    "mla_decode_attn": (ctypes.c_int, [ctypes.POINTER(mla_dims), _P, _P, _P, _I, _P, _I, _P,
                                       ctypes.c_float, _I, _P, _SZ, _P, _P, _P]),
    "mla_out_proj": (ctypes.c_int, [ctypes.POINTER(mla_dims), _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "mla_decode_attn_static_scratch": (ctypes.c_int, [ctypes.POINTER(mla_dims), _P, _P, _P, _I,
                                                      _P, _I, _P, ctypes.c_float, _I, _P, _P,
                                                      _P]),
    "mla_merge_partials": (ctypes.c_int, [ctypes.POINTER(mla_dims), _I, _P, _P, _P, _P, _P]),
    "mla_fold_weights": (ctypes.c_int, [ctypes.POINTER(mla_dims), _P, _P, _P, _P, _P, _P, _P]),
    "mla_step_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(mla_dims), _I, _I]),
    "mla_quantize_weights_fp8": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.c_int64, _P, _P, _P]),
    "mla_out_proj_fp8": (ctypes.c_int, [ctypes.POINTER(mla_dims), _P, _P, _P, _P, _P, _P, _P, _SZ,
                                        _P]),
    "mla_append_absorb_fp8": (ctypes.c_int, [ctypes.POINTER(mla_dims), _P, _P, _P, _P, _P, _P, _P,
                                             _P, _P, _P, _I, _P, _I, _P, _P, _P, _SZ, _P]),
    "mla_decode_step_host": (ctypes.c_int, [ctypes.POINTER(mla_dims), _I, ctypes.POINTER(mla_layer),
                                            _P, _P, _P, _P, _I, _P, _SZ, _P]),
    "mla_append_absorb_folded": (ctypes.c_int, [ctypes.POINTER(mla_dims), _P, _P, _P, _P, _P,
                                                _P, _I, _P, _I, _P, _P, _P, _SZ, _P]),
    "mla_out_proj_folded": (ctypes.c_int, [ctypes.POINTER(mla_dims), _P, _P, _P, _P, _SZ, _P]),
    "mla_get_status": (ctypes.c_int, [_P]),
    "mla_error_string": (ctypes.c_char_p, [ctypes.c_int]),
    "mla_error_detail": (ctypes.c_char_p, []),
    "mla_version": (ctypes.c_char_p, []),
    "mla_launch_count": (ctypes.c_uint64, []),
    "mla_set_profile_events": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p),
                                              ctypes.POINTER(ctypes.c_void_p), _I]),
    "mla_profile_events_used": (ctypes.c_int32, []),
}


def lib() -> ctypes.CDLL:
    """Load the CUDA library; fails loudly when it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m mla_latent_kv_37_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _error_string(code: int) -> str:
    try:
        return lib().mla_error_string(code).decode()
    except Exception:  # pragma: no cover
        return "?"


def _error_detail() -> str:
    try:
        return lib().mla_error_detail().decode()
    except Exception:  # pragma: no cover
        return ""


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, where: str):
    if rc != 0:
        raise MlaError(rc, where)


def _need(t, name, dtype=None, shape=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _elem(d: mla_dims):
    return torch.bfloat16 if d.dtype == MLA_BF16 else torch.float32


def mla_workspace_size(d: mla_dims, num_splits: int = 0) -> int:
    return int(lib().mla_workspace_size(ctypes.byref(d), num_splits))


def mla_cache_row_bytes(d: mla_dims) -> int:
    return int(lib().mla_cache_row_bytes(ctypes.byref(d)))


def workspace(d: mla_dims, num_splits: int = 0, device="cuda") -> torch.Tensor:
    n = mla_workspace_size(d, num_splits)
    if n == 0:
        raise MlaError(-2, "mla_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def mla_cache_append(d: mla_dims, h, w_dkv, w_kr, positions, page_table, cache_pool, ws=None,
                     stream=None):
    e = _elem(d)
    row = d.d_c + d.d_rope
    _need(h, "h", e, (d.batch, row) if w_dkv is None else (d.batch, d.d_model))
    _need(w_dkv, "w_dkv", e, (d.d_c, d.d_model))
    _need(w_kr, "w_kr", e, (d.d_rope, d.d_model))
    _need(positions, "positions", torch.int32, (d.batch,))
    _need(page_table, "page_table", torch.int32)
    _need(cache_pool, "cache_pool", e)
    _need(ws, "workspace", torch.uint8)
    rc = lib().mla_cache_append(ctypes.byref(d), _ptr(h), _ptr(w_dkv), _ptr(w_kr), _ptr(positions),
                                _ptr(page_table), page_table.shape[1], _ptr(cache_pool),
                                cache_pool.shape[0], _ptr(ws), 0 if ws is None else ws.numel(),
                                _stream(stream))
    _check(rc, "mla_cache_append")


def mla_absorb_q(d: mla_dims, h, w_q, w_uk, positions, q_cat, ws, q_lo=None, stream=None):
    e = _elem(d)
    H = d.n_heads
    _need(h, "h", e, (d.batch, d.d_model))
    _need(w_q, "w_q", e, (H * (d.d_nope + d.d_rope), d.d_model))
    _need(w_uk, "w_uk", e, (H * d.d_nope, d.d_c))
    _need(positions, "positions", torch.int32, (d.batch,))
    _need(q_cat, "q_cat", e, (d.batch, H, d.d_c + d.d_rope))
    _need(q_lo, "q_lo", torch.bfloat16, (d.batch, H, d.d_c + d.d_rope))
    _need(ws, "workspace", torch.uint8)
    rc = lib().mla_absorb_q(ctypes.byref(d), _ptr(h), _ptr(w_q), _ptr(w_uk), _ptr(positions),
                            _ptr(q_cat), _ptr(q_lo), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "mla_absorb_q")


def mla_append_absorb(d: mla_dims, h, w_dkv, w_kr, w_q, w_uk, positions, page_table, cache_pool,
                      q_cat, ws, q_lo=None, stream=None):
    """mla_cache_append + mla_absorb_q in one call (one shared projection launch)."""
    e = _elem(d)
    H = d.n_heads
    _need(h, "h", e, (d.batch, d.d_model))
    _need(w_dkv, "w_dkv", e, (d.d_c, d.d_model))
    _need(w_kr, "w_kr", e, (d.d_rope, d.d_model))
    _need(w_q, "w_q", e, (H * (d.d_nope + d.d_rope), d.d_model))
    _need(w_uk, "w_uk", e, (H * d.d_nope, d.d_c))
    _need(positions, "positions", torch.int32, (d.batch,))
    _need(page_table, "page_table", torch.int32)
    _need(cache_pool, "cache_pool", e)
    _need(q_cat, "q_cat", e, (d.batch, H, d.d_c + d.d_rope))
    _need(q_lo, "q_lo", torch.bfloat16, (d.batch, H, d.d_c + d.d_rope))
    _need(ws, "workspace", torch.uint8)
    rc = lib().mla_append_absorb(ctypes.byref(d), _ptr(h), _ptr(w_dkv), _ptr(w_kr), _ptr(w_q),
                                 _ptr(w_uk), _ptr(positions), _ptr(page_table),
                                 page_table.shape[1], _ptr(cache_pool), cache_pool.shape[0],
                                 _ptr(q_cat), _ptr(q_lo), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "mla_append_absorb")


def mla_decode_attn(d: mla_dims, q_cat, cache_pool, page_table, seq_lens, o_lat, ws, lse=None,
                    q_lo=None, softmax_scale: float = 0.0, num_splits: int = 0, stream=None):
    e = _elem(d)
    H = d.n_heads
    _need(q_cat, "q_cat", e, (d.batch, H, d.d_c + d.d_rope))
    _need(cache_pool, "cache_pool", e)
    _need(page_table, "page_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32, (d.batch,))
    _need(o_lat, "o_lat", torch.float32, (d.batch, H, d.d_c))
    _need(lse, "lse", torch.float32, (d.batch, H))
    _need(q_lo, "q_lo", torch.bfloat16, (d.batch, H, d.d_c + d.d_rope))
    _need(ws, "workspace", torch.uint8)
    rc = lib().mla_decode_attn(ctypes.byref(d), _ptr(q_cat), _ptr(q_lo), _ptr(cache_pool),
                               cache_pool.shape[0], _ptr(page_table), page_table.shape[1],
                               _ptr(seq_lens), float(softmax_scale), int(num_splits), _ptr(ws),
                               ws.numel(), _ptr(o_lat), _ptr(lse), _stream(stream))
    _check(rc, "mla_decode_attn")


def mla_decode_attn_static_scratch(d: mla_dims, q_cat, cache_pool, page_table, seq_lens, o_lat,
                                   lse=None, softmax_scale: float = 0.0, num_splits: int = 0,
                                   stream=None):
    """mla_decode_attn without a workspace: the library's own fixed scratch array is used, for
    callers that cannot allocate device memory (see include/mla.h)."""
    e = _elem(d)
    H = d.n_heads
    _need(q_cat, "q_cat", e, (d.batch, H, d.d_c + d.d_rope))
    _need(cache_pool, "cache_pool", e)
    _need(page_table, "page_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32, (d.batch,))
    _need(o_lat, "o_lat", torch.float32, (d.batch, H, d.d_c))
    _need(lse, "lse", torch.float32, (d.batch, H))
    rc = lib().mla_decode_attn_static_scratch(ctypes.byref(d), _ptr(q_cat), None,
                                              _ptr(cache_pool), cache_pool.shape[0],
                                              _ptr(page_table), page_table.shape[1],
                                              _ptr(seq_lens), float(softmax_scale),
                                              int(num_splits), _ptr(o_lat), _ptr(lse),
                                              _stream(stream))
    _check(rc, "mla_decode_attn_static_scratch")


def mla_out_proj(d: mla_dims, o_lat, w_uv, ws, w_o=None, o_heads=None, out=None, stream=None):
    e = _elem(d)
    H = d.n_heads
    _need(o_lat, "o_lat", torch.float32, (d.batch, H, d.d_c))
    _need(w_uv, "w_uv", e, (H * d.d_v, d.d_c))
    _need(w_o, "w_o", e, (d.d_model, H * d.d_v))
    _need(o_heads, "o_heads", e, (d.batch, H, d.d_v))
    _need(out, "out", e, (d.batch, d.d_model))
    _need(ws, "workspace", torch.uint8)
    rc = lib().mla_out_proj(ctypes.byref(d), _ptr(o_lat), _ptr(w_uv), _ptr(w_o), _ptr(o_heads),
                            _ptr(out), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "mla_out_proj")


def layer_structs(d: mla_dims, layers):
    """ctypes array of mla_layer for step layers (objects with the Layer fields; a layer with
    `e4m3` copies passes its codes and row scales instead of the bf16 W_DKV, W_KR, W_Q, W_O)."""
    e = _elem(d)
    arr = (mla_layer * len(layers))()
    for i, ly in enumerate(layers):
        H = d.n_heads
        shapes = {"w_dkv": (d.d_c, d.d_model), "w_kr": (d.d_rope, d.d_model),
                  "w_q": (H * (d.d_nope + d.d_rope), d.d_model), "w_o": (d.d_model, H * d.d_v)}
        if ly.w_o is None:
            raise ValueError("w_o is required: the step's result is out")
        q = getattr(ly, "e4m3", None)
        ptrs, scales = {}, {}
        for n, shp in shapes.items():
            if q is not None:
                codes, scale = q[n]
                _need(codes, n + " codes", torch.uint8, fp8_codes_shape(*shp))
                _need(scale, n + " scale", torch.float32, (shp[0],))
                ptrs[n], scales[n] = _ptr(codes), _ptr(scale)
            else:
                _need(getattr(ly, n), n, e, shp)
                ptrs[n], scales[n] = _ptr(getattr(ly, n)), None
        _need(ly.w_uk, "w_uk", e, (H * d.d_nope, d.d_c))
        _need(ly.w_uv, "w_uv", e, (H * d.d_v, d.d_c))
        _need(ly.pool, "cache_pool", e)
        _need(ly.page_table, "page_table", torch.int32)
        arr[i] = mla_layer(ptrs["w_dkv"], ptrs["w_kr"], ptrs["w_q"], _ptr(ly.w_uk),
                           _ptr(ly.w_uv), ptrs["w_o"], _ptr(ly.pool), ly.pool.shape[0],
                           _ptr(ly.page_table), ly.page_table.shape[1], scales["w_dkv"],
                           scales["w_kr"], scales["w_q"], scales["w_o"])
    return arr


def step_workspace(d: mla_dims, n_layers: int, num_splits: int = 0, device="cuda"):
    n = lib().mla_step_workspace_size(ctypes.byref(d), n_layers, num_splits)
    if n == 0:
        raise MlaError(-2, "mla_step_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def mla_decode_step_host(d: mla_dims, layer_array, h_host, positions_host, seq_lens_host,
                         out_host, ws, num_splits: int = 0, stream=None):
    """One decode step over len(layer_array) layers from host buffers (the native executor)."""
    L = len(layer_array)
    e = _elem(d)
    for t, name, dt, shape in ((h_host, "h_host", e, (L, d.batch, d.d_model)),
                               (positions_host, "positions_host", torch.int32, (d.batch,)),
                               (seq_lens_host, "seq_lens_host", torch.int32, (d.batch,)),
                               (out_host, "out_host", e, (L, d.batch, d.d_model))):
        if t.is_cuda or not t.is_contiguous() or t.dtype != dt or tuple(t.shape) != shape:
            raise ValueError(f"{name} must be a contiguous host tensor {dt} {shape}")
    _need(ws, "workspace", torch.uint8)
    rc = lib().mla_decode_step_host(ctypes.byref(d), L, layer_array, h_host.data_ptr(),
                                    positions_host.data_ptr(), seq_lens_host.data_ptr(),
                                    out_host.data_ptr(), num_splits, _ptr(ws), ws.numel(),
                                    _stream(stream))
    _check(rc, "mla_decode_step_host")


def mla_quantize_weights_fp8(w, codes, scale, stream=None):
    """E4M3 storage of a bf16 matrix w [rows, cols]: scale [rows] fp32 and codes uint8 in
    128 x 128 tiles, [round_up(rows, 128), cols] bytes (see mla_quantize_weights_fp8 in mla.h)."""
    _need(w, "w", torch.bfloat16)
    if w.dim() != 2:
        raise ValueError("w must be a matrix")
    rows, cols = w.shape
    _need(codes, "codes", torch.uint8, fp8_codes_shape(rows, cols))
    _need(scale, "scale", torch.float32, (rows,))
    rc = lib().mla_quantize_weights_fp8(_ptr(w), rows, cols, _ptr(codes), _ptr(scale),
                                        _stream(stream))
    _check(rc, "mla_quantize_weights_fp8")


def fp8_codes_shape(rows, cols):
    """Shape of the E4M3 code buffer of a [rows, cols] matrix (128 x 128 tiles)."""
    return ((rows + 127) // 128 * 128, cols)


def fp8_codes_rows(codes, rows, cols):
    """The codes of a tiled E4M3 buffer rearranged as the [rows, cols] matrix (a layout change
    on the tensor's device, for inspection and host-side checks)."""
    rt = codes.shape[0] // 128
    t = codes.reshape(rt, cols // 128, 128, 128).permute(0, 2, 1, 3).reshape(rt * 128, cols)
    return t[:rows]


def mla_append_absorb_fp8(d: mla_dims, h, w_dkv, w_kr, w_q, w_uk, positions, page_table,
                          cache_pool, q_cat, ws, q_lo=None, stream=None):
    """mla_append_absorb with W_DKV, W_KR, W_Q given as (codes, scale) pairs from
    mla_quantize_weights_fp8 (bf16 path); W_UK stays bf16."""
    H = d.n_heads
    m_q = H * (d.d_nope + d.d_rope)
    pairs = (("w_dkv", w_dkv, d.d_c), ("w_kr", w_kr, d.d_rope), ("w_q", w_q, m_q))
    for name, (codes, scale), rows in pairs:
        _need(codes, name + " codes", torch.uint8, fp8_codes_shape(rows, d.d_model))
        _need(scale, name + " scale", torch.float32, (rows,))
    _need(h, "h", torch.bfloat16, (d.batch, d.d_model))
    _need(w_uk, "w_uk", torch.bfloat16, (H * d.d_nope, d.d_c))
    _need(positions, "positions", torch.int32, (d.batch,))
    _need(page_table, "page_table", torch.int32)
    _need(cache_pool, "cache_pool", torch.bfloat16)
    _need(q_cat, "q_cat", torch.bfloat16, (d.batch, H, d.d_c + d.d_rope))
    _need(q_lo, "q_lo", torch.bfloat16, (d.batch, H, d.d_c + d.d_rope))
    _need(ws, "workspace", torch.uint8)
    rc = lib().mla_append_absorb_fp8(
        ctypes.byref(d), _ptr(h), _ptr(w_dkv[0]), _ptr(w_dkv[1]), _ptr(w_kr[0]), _ptr(w_kr[1]),
        _ptr(w_q[0]), _ptr(w_q[1]), _ptr(w_uk), _ptr(positions), _ptr(page_table),
        page_table.shape[1], _ptr(cache_pool), cache_pool.shape[0], _ptr(q_cat), _ptr(q_lo),
        _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "mla_append_absorb_fp8")


def mla_out_proj_fp8(d: mla_dims, o_lat, w_uv, w_o_codes, w_o_scale, out, ws, o_heads=None,
                     stream=None):
    """mla_out_proj with W_O stored as E4M3 codes (tiled, as mla_quantize_weights_fp8 writes
    them) and row scales (bf16 path)."""
    H = d.n_heads
    _need(o_lat, "o_lat", torch.float32, (d.batch, H, d.d_c))
    _need(w_uv, "w_uv", torch.bfloat16, (H * d.d_v, d.d_c))
    _need(w_o_codes, "w_o_codes", torch.uint8, fp8_codes_shape(d.d_model, H * d.d_v))
    _need(w_o_scale, "w_o_scale", torch.float32, (d.d_model,))
    _need(o_heads, "o_heads", torch.bfloat16, (d.batch, H, d.d_v))
    _need(out, "out", torch.bfloat16, (d.batch, d.d_model))
    _need(ws, "workspace", torch.uint8)
    rc = lib().mla_out_proj_fp8(ctypes.byref(d), _ptr(o_lat), _ptr(w_uv), _ptr(w_o_codes),
                                _ptr(w_o_scale), _ptr(o_heads), _ptr(out), _ptr(ws), ws.numel(),
                                _stream(stream))
    _check(rc, "mla_out_proj_fp8")


def fold_shapes(d: mla_dims):
    """Shapes of the folded weights: (w_qf [H, d_c + d_R, D], w_of [D, H * d_c])."""
    H = d.n_heads
    return (H, d.d_c + d.d_rope, d.d_model), (d.d_model, H * d.d_c)


def mla_fold_weights(d: mla_dims, w_q=None, w_uk=None, w_uv=None, w_o=None, w_qf=None,
                     w_of=None, stream=None):
    """The one-time folding of the folded execution mode (bf16): W_UK into W_Q, W_UV into W_O."""
    e = _elem(d)
    H = d.n_heads
    sq, so = fold_shapes(d)
    _need(w_q, "w_q", e, (H * (d.d_nope + d.d_rope), d.d_model))
    _need(w_uk, "w_uk", e, (H * d.d_nope, d.d_c))
    _need(w_uv, "w_uv", e, (H * d.d_v, d.d_c))
    _need(w_o, "w_o", e, (d.d_model, H * d.d_v))
    _need(w_qf, "w_qf", e, sq)
    _need(w_of, "w_of", e, so)
    rc = lib().mla_fold_weights(ctypes.byref(d), _ptr(w_q), _ptr(w_uk), _ptr(w_uv), _ptr(w_o),
                                _ptr(w_qf), _ptr(w_of), _stream(stream))
    _check(rc, "mla_fold_weights")


def mla_append_absorb_folded(d: mla_dims, h, w_dkv, w_kr, w_qf, positions, page_table,
                             cache_pool, q_cat, ws, q_lo=None, stream=None):
    """Cache append and the folded query in one projection launch (bf16)."""
    e = _elem(d)
    H = d.n_heads
    _need(h, "h", e, (d.batch, d.d_model))
    _need(w_dkv, "w_dkv", e, (d.d_c, d.d_model))
    _need(w_kr, "w_kr", e, (d.d_rope, d.d_model))
    _need(w_qf, "w_qf", e, fold_shapes(d)[0])
    _need(positions, "positions", torch.int32, (d.batch,))
    _need(page_table, "page_table", torch.int32)
    _need(cache_pool, "cache_pool", e)
    _need(q_cat, "q_cat", e, (d.batch, H, d.d_c + d.d_rope))
    _need(q_lo, "q_lo", torch.bfloat16, (d.batch, H, d.d_c + d.d_rope))
    _need(ws, "workspace", torch.uint8)
    rc = lib().mla_append_absorb_folded(ctypes.byref(d), _ptr(h), _ptr(w_dkv), _ptr(w_kr),
                                        _ptr(w_qf), _ptr(positions), _ptr(page_table),
                                        page_table.shape[1], _ptr(cache_pool),
                                        cache_pool.shape[0], _ptr(q_cat), _ptr(q_lo), _ptr(ws),
                                        ws.numel(), _stream(stream))
    _check(rc, "mla_append_absorb_folded")


def mla_out_proj_folded(d: mla_dims, o_lat, w_of, out, ws, stream=None):
    """out = W_OF o_lat with the folded output weights (bf16)."""
    e = _elem(d)
    _need(o_lat, "o_lat", torch.float32, (d.batch, d.n_heads, d.d_c))
    _need(w_of, "w_of", e, fold_shapes(d)[1])
    _need(out, "out", e, (d.batch, d.d_model))
    _need(ws, "workspace", torch.uint8)
    rc = lib().mla_out_proj_folded(ctypes.byref(d), _ptr(o_lat), _ptr(w_of), _ptr(out), _ptr(ws),
                                   ws.numel(), _stream(stream))
    _check(rc, "mla_out_proj_folded")


def mla_merge_partials(d: mla_dims, part_o, part_lse, o_lat, lse=None, stream=None):
    """Merge partial attention results [n, B, H, 512] / [n, B, H] into o_lat / lse."""
    n = part_o.shape[0]
    _need(part_o, "part_o", torch.float32, (n, d.batch, d.n_heads, d.d_c))
    _need(part_lse, "part_lse", torch.float32, (n, d.batch, d.n_heads))
    _need(o_lat, "o_lat", torch.float32, (d.batch, d.n_heads, d.d_c))
    _need(lse, "lse", torch.float32, (d.batch, d.n_heads))
    rc = lib().mla_merge_partials(ctypes.byref(d), n, _ptr(part_o), _ptr(part_lse), _ptr(o_lat),
                                  _ptr(lse), _stream(stream))
    _check(rc, "mla_merge_partials")


def mla_get_status(stream=None) -> int:
    rc = lib().mla_get_status(_stream(stream))
    if rc < 0:
        raise MlaError(rc, "mla_get_status")
    return rc


def version() -> str:
    return lib().mla_version().decode()


def mla_launch_count() -> int:
    return int(lib().mla_launch_count())


_prof_keep = None


def mla_set_profile_events(begin, end) -> None:
    """begin/end: equal-length lists of torch.cuda.Event(enable_timing=True)."""
    global _prof_keep
    n = len(begin)
    assert len(end) == n
    for e in list(begin) + list(end):
        if e.cuda_event == 0:  # events are created lazily by torch
            e.record()
    arr_b = (ctypes.c_void_p * max(n, 1))(*[e.cuda_event for e in begin])
    arr_e = (ctypes.c_void_p * max(n, 1))(*[e.cuda_event for e in end])
    _prof_keep = (arr_b, arr_e, begin, end)
    _check(lib().mla_set_profile_events(arr_b, arr_e, n), "mla_set_profile_events")


def mla_profile_events_used() -> int:
    return int(lib().mla_profile_events_used())
