"""Python binding of libmla (include/mla.h): MLA decode over a paged latent KV cache
on NVIDIA B200 (sm_100a).

The binding only marshals arguments: it turns torch tensors into device
pointers and sizes and calls the C entry points of the same names.  Every step
of the decode path runs in the library's CUDA kernels; there is no other
implementation behind these functions.  If ``libmla.so`` has not been built,
importing this package raises ``ImportError``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "MLAError", "Handle", "lib", "LIB_PATH",
    "mla_create", "mla_destroy", "mla_cache_append", "mla_kv_project_append", "mla_absorb_q",
    "mla_decode", "mla_decode_partial", "mla_decode_combine", "mla_decode_auto_splits",
    "mla_decode_noalloc",
    "mla_decode_workspace_bytes", "mla_out_proj", "mla_out_proj_workspace_bytes",
    "mla_last_device_error", "mla_set_wait_limit", "mla_set_launch_overlap", "mla_status_string",
    "mla_launch_count", "mla_combine_out_proj", "mla_pack_w_o", "mla_set_w_o_layout",
    "MLA_BF16", "MLA_FP8_E4M3", "MLA_FP32", "EXPORTED_SYMBOLS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla.so")

MLA_BF16, MLA_FP8_E4M3, MLA_FP32 = 0, 1, 2
_DTYPES = {"bf16": MLA_BF16, "fp8_e4m3": MLA_FP8_E4M3, "fp32": MLA_FP32}

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libmla.so is not built ({LIB_PATH}); run `python mla_latent_kv_19_b200/build.py`")

lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int32
_SZ = ctypes.c_size_t


class MlaConfig(ctypes.Structure):
    _fields_ = [
        ("num_heads", ctypes.c_int32), ("d_c", ctypes.c_int32), ("d_r", ctypes.c_int32),
        ("d_nope", ctypes.c_int32), ("d_v", ctypes.c_int32), ("d_model", ctypes.c_int32),
        ("block_size", ctypes.c_int32), ("act_dtype", ctypes.c_int32),
        ("cache_dtype", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
        ("rope_base", ctypes.c_float), ("max_position", ctypes.c_int32),
    ]


_SIGS = {
    "mla_create": (ctypes.c_int, [ctypes.POINTER(MlaConfig), ctypes.POINTER(_P)]),
    "mla_destroy": (ctypes.c_int, [_P]),
    "mla_cache_row_bytes": (_SZ, [_P]),
    "mla_cache_scale_bytes": (_SZ, [_P]),
    "mla_cache_append": (ctypes.c_int, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _P, _P, _I, _P]),
    "mla_kv_project_append": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I, _P, _I, _I, _P, _P, _I, _P]),
    "mla_absorb_q": (ctypes.c_int, [_P, _P, _P, _P, _P, _I, _P, _P]),
    "mla_decode_auto_splits": (ctypes.c_int32, [_P, _I, _I]),
    "mla_decode_workspace_bytes": (_SZ, [_P, _I, _I, _I]),
    "mla_decode": (ctypes.c_int, [_P, _P, _P, _P, _I, _P, _I, _P, _I, _I, _I, _P, _SZ, _P, _P, _P]),
    "mla_decode_partial": (ctypes.c_int, [_P, _P, _P, _P, _I, _P, _I, _P, _I, _I, _I, _P, _SZ, _P]),
    "mla_decode_combine": (ctypes.c_int, [_P, _I, _I, _I, _P, _SZ, _P, _P, _P]),
    "mla_decode_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _I, _P, _I, _P, _I, _I, _I, _P, _P, _P]),
    "mla_out_proj_workspace_bytes": (_SZ, [_P, _I]),
    "mla_out_proj": (ctypes.c_int, [_P, _P, _P, _P, _I, _P, _SZ, _P, _P, _P]),
    "mla_combine_out_proj": (ctypes.c_int, [_P, _I, _I, _I, _P, _SZ, _P, _P, _P, _SZ, _P, _P, _P, _P, _P]),
    "mla_last_device_error": (ctypes.c_int, [_P, _P]),
    "mla_set_wait_limit": (ctypes.c_int, [_P, ctypes.c_uint32]),
    "mla_set_launch_overlap": (ctypes.c_int, [_P, ctypes.c_int]),
    "mla_pack_w_o": (ctypes.c_int, [_P, _P, _P, _P]),
    "mla_set_w_o_layout": (ctypes.c_int, [_P, ctypes.c_int]),
    "mla_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "mla_launch_count": (ctypes.c_uint64, []),
}
EXPORTED_SYMBOLS = tuple(_SIGS)

for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class MLAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {mla_status_string(status)} ({status})")


def mla_status_string(status: int) -> str:
    return lib.mla_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise MLAError(fn, status)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libmla must be contiguous")
    return t.data_ptr()


def _num_blocks(h: "Handle", cache) -> int:
    """Pages in a cache tensor of any shape: its elements / (block_size * (d_c + d_r))."""
    per_page = h.cfg.block_size * (h.cfg.d_c + h.cfg.d_r)
    n, rem = divmod(cache.numel(), per_page)
    if rem or n == 0:
        raise ValueError(f"cache of {cache.numel()} elements is not a whole number of "
                         f"{per_page}-element pages")
    return n


def _scale_ptr(h: "Handle", cache, cache_scale) -> Optional[int]:
    """Pointer of an fp8 cache's per-token scales, after checking that it holds
    one fp32 per cache row (the kernels read a page's scales by page index)."""
    if cache_scale is None:
        return None
    rows = _num_blocks(h, cache) * h.cfg.block_size
    if cache_scale.dtype != torch.float32 or cache_scale.numel() < rows:
        raise ValueError(f"cache_scale must hold {rows} fp32 values (one per cache row), "
                         f"got {cache_scale.numel()} of {cache_scale.dtype}")
    return _ptr(cache_scale)


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class Handle:
    """Owns an ``mla_handle_t`` created on the current CUDA device."""

    def __init__(self, *, num_heads: int, d_c: int, d_r: int, d_nope: int, d_v: int, d_model: int,
                 block_size: int = 64, act_dtype: str = "bf16", cache_dtype: str = "bf16",
                 softmax_scale: float, rope_base: float = 10000.0, max_position: int = 131072 + 64):
        cfg = MlaConfig(num_heads, d_c, d_r, d_nope, d_v, d_model, block_size,
                        _DTYPES[act_dtype], _DTYPES[cache_dtype], softmax_scale, rope_base,
                        max_position)
        self.cfg = cfg
        self.act_dtype, self.cache_dtype = act_dtype, cache_dtype
        h = _P()
        _check("mla_create", lib.mla_create(ctypes.byref(cfg), ctypes.byref(h)))
        self._h = h

    @property
    def ptr(self):
        return self._h

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib.mla_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def mla_create(**kw) -> Handle:
    return Handle(**kw)


def mla_destroy(h: Handle) -> None:
    h.close()


def mla_cache_append(h: Handle, c_kv, k_r, pos, block_table, cache, cache_scale=None,
                     seq_idx=None, batch: Optional[int] = None, stream=None) -> None:
    n = pos.shape[0]
    batch = block_table.shape[0] if batch is None else batch
    _check("mla_cache_append", lib.mla_cache_append(
        h.ptr, _ptr(c_kv), _ptr(k_r), _ptr(seq_idx), _ptr(pos), n, _ptr(block_table),
        block_table.shape[1], batch, _ptr(cache), _scale_ptr(h, cache, cache_scale), _num_blocks(h, cache), _stream(stream)))


def mla_kv_project_append(h: Handle, x, w_dkv, w_kr, pos, block_table, cache, cache_scale=None,
                          seq_idx=None, batch: Optional[int] = None, stream=None) -> None:
    n = pos.shape[0]
    batch = block_table.shape[0] if batch is None else batch
    _check("mla_kv_project_append", lib.mla_kv_project_append(
        h.ptr, _ptr(x), _ptr(w_dkv), _ptr(w_kr), _ptr(seq_idx), _ptr(pos), n, _ptr(block_table),
        block_table.shape[1], batch, _ptr(cache), _scale_ptr(h, cache, cache_scale), _num_blocks(h, cache), _stream(stream)))


def mla_absorb_q(h: Handle, q_nope, q_pe, pos, w_uk, q_lat, stream=None) -> None:
    _check("mla_absorb_q", lib.mla_absorb_q(
        h.ptr, _ptr(q_nope), _ptr(q_pe), _ptr(pos), _ptr(w_uk), q_nope.shape[0], _ptr(q_lat),
        _stream(stream)))


def mla_decode_auto_splits(h: Handle, batch: int, max_seq_len: int) -> int:
    return int(lib.mla_decode_auto_splits(h.ptr, batch, max_seq_len))


def mla_decode_workspace_bytes(h: Handle, batch: int, num_splits: int, max_seq_len: int) -> int:
    return int(lib.mla_decode_workspace_bytes(h.ptr, batch, num_splits, max_seq_len))


def mla_decode(h: Handle, q_lat, cache, cache_scale, block_table, seq_lens, max_seq_len: int,
               num_splits: int, workspace, o_lat, lse=None, stream=None) -> None:
    _check("mla_decode", lib.mla_decode(
        h.ptr, _ptr(q_lat), _ptr(cache), _scale_ptr(h, cache, cache_scale), _num_blocks(h, cache), _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), seq_lens.shape[0], max_seq_len, num_splits,
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(o_lat), _ptr(lse),
        _stream(stream)))


def mla_decode_partial(h: Handle, q_lat, cache, cache_scale, block_table, seq_lens,
                       max_seq_len: int, num_splits: int, workspace, stream=None) -> None:
    _check("mla_decode_partial", lib.mla_decode_partial(
        h.ptr, _ptr(q_lat), _ptr(cache), _scale_ptr(h, cache, cache_scale), _num_blocks(h, cache), _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), seq_lens.shape[0], max_seq_len, num_splits,
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def mla_decode_combine(h: Handle, batch: int, max_seq_len: int, num_splits: int, workspace, o_lat,
                       lse=None, stream=None) -> None:
    _check("mla_decode_combine", lib.mla_decode_combine(
        h.ptr, batch, max_seq_len, num_splits, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(o_lat), _ptr(lse), _stream(stream)))


def mla_decode_noalloc(h: Handle, q_lat, cache, cache_scale, block_table, seq_lens,
                       max_seq_len: int, num_splits: int, o_lat, lse=None, stream=None) -> None:
    """mla_decode without a caller workspace: the split partials live in a
    fixed 32 MiB device array inside the library (for callers that cannot
    allocate device memory).  Overlapping calls on one device race on it."""
    _check("mla_decode_noalloc", lib.mla_decode_noalloc(
        h.ptr, _ptr(q_lat), _ptr(cache), _scale_ptr(h, cache, cache_scale), _num_blocks(h, cache), _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), seq_lens.shape[0], max_seq_len, num_splits,
        _ptr(o_lat), _ptr(lse), _stream(stream)))


def mla_out_proj_workspace_bytes(h: Handle, batch: int) -> int:
    return int(lib.mla_out_proj_workspace_bytes(h.ptr, batch))


def mla_out_proj(h: Handle, o_lat, w_uv, w_o, workspace, y, o_out=None, stream=None) -> None:
    _check("mla_out_proj", lib.mla_out_proj(
        h.ptr, _ptr(o_lat), _ptr(w_uv), _ptr(w_o), o_lat.shape[0], _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(y), _ptr(o_out), _stream(stream)))


def mla_combine_out_proj(h: Handle, batch: int, max_seq_len: int, num_splits: int, workspace, w_uv, w_o,
                         op_workspace, o_lat, y, lse=None, o_out=None, stream=None) -> None:
    _check("mla_combine_out_proj", lib.mla_combine_out_proj(
        h.ptr, batch, max_seq_len, num_splits, _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(w_uv), _ptr(w_o), _ptr(op_workspace), op_workspace.numel() * op_workspace.element_size(),
        _ptr(o_lat), _ptr(lse), _ptr(y), _ptr(o_out), _stream(stream)))


def mla_last_device_error(h: Handle, stream=None) -> int:
    return int(lib.mla_last_device_error(h.ptr, _stream(stream)))


def mla_launch_count() -> int:
    return int(lib.mla_launch_count())


def mla_set_wait_limit(h: Handle, limit: int) -> None:
    _check("mla_set_wait_limit", lib.mla_set_wait_limit(h.ptr, limit))


def mla_pack_w_o(h: Handle, w_o, w_o_tiled, stream=None) -> None:
    """w_o_tiled <- W_O in tile-major order ([d_model/128][H*d_v/64][128][64])."""
    _check("mla_pack_w_o", lib.mla_pack_w_o(h.ptr, _ptr(w_o), _ptr(w_o_tiled), _stream(stream)))


def mla_set_w_o_layout(h: Handle, tiled: bool) -> None:
    """Whether later output projections on h read a tile-major w_o."""
    _check("mla_set_w_o_layout", lib.mla_set_w_o_layout(h.ptr, 1 if tiled else 0))


def mla_set_launch_overlap(h: Handle, enable: bool) -> None:
    """Launch this handle's kernels as programmatic dependents of the kernel
    before them on the stream (weights are then read before that kernel ends)."""
    _check("mla_set_launch_overlap", lib.mla_set_launch_overlap(h.ptr, 1 if enable else 0))
