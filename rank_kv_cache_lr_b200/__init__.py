"""Python binding of the low-rank KV-cache decode library (C ABI in include/lr_kv.h).

Argument marshalling only: every step of the path runs in the CUDA library
`_lib/liblrkv.so`.  Tensors are torch CUDA tensors (device memory and streams
come from PyTorch); they are checked for device, dtype, shape and contiguity
and passed by pointer.  There is no fallback: if the library is missing,
importing this package raises.

Functions keep the C names: lr_cache_create, lr_cache_destroy, lr_kv_append, lr_decode_step,
lr_kv_append_latent, lr_attn_decode, lr_basis_sync, lr_basis_update, lr_cache_get_len,
lr_cache_truncate, lr_cache_view_get, lr_cache_set_path, lr_cache_plan,
lr_plan_decode, lr_cache_set_kernel_events, lr_cache_set_trace, lr_device_error, lr_abi_struct_sizes,
lr_status_string, lr_launch_count, lr_attn_decode_noalloc, lr_cache_set_wait_limit,
lr_debug_inject_fault, lr_attn_decode_varlen, lr_attn_decode_partial, lr_merge_partials,
lr_kv_prefill, lr_cache_set_block_table, lr_cache_set_block_table_device, lr_kv_append_rows.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "liblrkv.so")

LR_OK, LR_ERR_INVALID_ARG, LR_ERR_UNSUPPORTED, LR_ERR_CAPACITY = 0, 1, 2, 3
LR_ERR_CUDA, LR_ERR_OOM, LR_ERR_TIMEOUT = 4, 5, 6
LR_F32, LR_BF16 = 0, 1
LR_PATH_AUTO, LR_PATH_SIMT, LR_PATH_TC = 0, 1, 2


class lr_cache_desc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("rank_k", ctypes.c_int32), ("rank_v", ctypes.c_int32),
                ("capacity", ctypes.c_int32), ("window", ctypes.c_int32),
                ("quant_bits", ctypes.c_int32), ("quant_group", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("rope_in_kernel", ctypes.c_int32),
                ("rope_theta", ctypes.c_double), ("softmax_scale", ctypes.c_float),
                ("latent_groups", ctypes.c_int32), ("page_tokens", ctypes.c_int32),
                ("n_pages", ctypes.c_int32), ("reserved", ctypes.c_int32 * 2)]


class lr_cache_view(ctypes.Structure):
    _fields_ = [("z_k", ctypes.c_void_p), ("z_v", ctypes.c_void_p),
                ("codes_k", ctypes.c_void_p), ("codes_v", ctypes.c_void_p),
                ("params_k", ctypes.c_void_p), ("params_v", ctypes.c_void_p),
                ("win_k", ctypes.c_void_p), ("win_v", ctypes.c_void_p),
                ("A_k", ctypes.c_void_p), ("B_k", ctypes.c_void_p),
                ("A_v", ctypes.c_void_p), ("B_v", ctypes.c_void_p),
                ("groups_k", ctypes.c_int32), ("groups_v", ctypes.c_int32),
                ("capacity", ctypes.c_int32), ("window_slots", ctypes.c_int32),
                ("int4_blocks", ctypes.c_int32), ("n_pages", ctypes.c_int32)]


class lr_plan(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("n_splits", ctypes.c_int32),
                ("tile_tokens", ctypes.c_int32), ("split_tokens", ctypes.c_int32),
                ("ctas", ctypes.c_int32)]


class LRError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_name(status)}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"CUDA library not built: {LIB_PATH} is missing "
                          "(run `python -c 'import __graft_entry__ as g; g.build()'`)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, st = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int
    sig = {
        "lr_cache_create": [ctypes.POINTER(lr_cache_desc), vp, vp, vp, vp, vp, ctypes.POINTER(vp)],
        "lr_cache_destroy": [vp],
        "lr_kv_append": [vp, vp, vp, vp],
        "lr_kv_append_latent": [vp, vp, vp, i32, vp],
        "lr_attn_decode": [vp, vp, vp, vp, vp],
        "lr_decode_step": [vp, vp, vp, vp, vp, vp, vp],
        "lr_basis_sync": [vp, vp, vp, vp, vp, vp, vp, vp],
        "lr_basis_update": [vp, i32, vp, i32, vp, vp, vp, vp, vp],
        "lr_cache_get_len": [vp, ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(i32)],
        "lr_cache_truncate": [vp, i32],
        "lr_cache_view_get": [vp, ctypes.POINTER(lr_cache_view)],
        "lr_cache_set_block_table": [vp, vp, vp],
        "lr_cache_set_block_table_device": [vp, vp, vp],
        "lr_cache_set_path": [vp, i32, i32],
        "lr_cache_plan": [vp, ctypes.POINTER(lr_plan)],
        "lr_plan_decode": [ctypes.POINTER(lr_cache_desc), i32, i32, i32, i32, ctypes.POINTER(lr_plan)],
        "lr_device_error": [vp, ctypes.POINTER(i32)],
        "lr_cache_set_kernel_events": [vp, vp, vp],
        "lr_cache_set_trace": [vp, vp, ctypes.c_int64],
        "lr_cache_set_wait_limit": [vp, ctypes.c_int64],
        "lr_attn_decode_varlen": [vp, vp, vp, vp, vp, vp],
        "lr_attn_decode_partial": [vp, vp, vp, vp, vp],
        "lr_kv_prefill": [vp, vp, vp, i32, vp],
        "lr_kv_append_rows": [vp, vp, vp, vp, i32, vp],
        "lr_merge_partials": [vp, i32, vp, vp, vp, vp, vp],
        "lr_debug_inject_fault": [i32, ctypes.c_int64],
        "lr_attn_decode_noalloc": [ctypes.POINTER(lr_cache_desc), i32, vp, vp, vp, vp, vp, vp, vp, vp],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = st
    lib.lr_status_string.argtypes = [st]
    lib.lr_status_string.restype = ctypes.c_char_p
    lib.lr_abi_struct_sizes.argtypes = [ctypes.POINTER(i32)] * 3
    lib.lr_abi_struct_sizes.restype = None
    lib.lr_launch_count.argtypes = []
    lib.lr_launch_count.restype = ctypes.c_int64
    return lib


_lib = _load()


def status_name(status: int) -> str:
    return _lib.lr_status_string(int(status)).decode()


lr_status_string = status_name


def _check(status: int, where: str) -> None:
    if status != LR_OK:
        raise LRError(status, where)


def lr_launch_count() -> int:
    return int(_lib.lr_launch_count())


def make_desc(batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int, rank_k: int,
              rank_v: int, capacity: int, window: int = 0, quant_bits: int = 0,
              dtype: int = LR_BF16, rope_in_kernel: int = 0, rope_theta: float = 1e6,
              softmax_scale: float = 0.0, quant_group: int = 32,
              latent_groups: int = 0, page_tokens: int = 0, n_pages: int = 0) -> lr_cache_desc:
    return lr_cache_desc(batch, n_q_heads, n_kv_heads, head_dim, rank_k, rank_v, capacity,
                         window, quant_bits, quant_group, dtype, rope_in_kernel, rope_theta,
                         softmax_scale, latent_groups, page_tokens, n_pages)


# ---------------------------------------------------------------------------
# tensor marshalling
# ---------------------------------------------------------------------------

def _torch_dtype(code: int):
    import torch
    return torch.bfloat16 if code == LR_BF16 else torch.float32


def _ptr(t, dtype=None, shape=None, name="tensor", allow_none=False):
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    if not getattr(t, "is_cuda", False):
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class Cache:
    """Handle of one lr_cache (one layer).  Holds the description for shape checks."""

    def __init__(self, handle: ctypes.c_void_p, desc: lr_cache_desc):
        self.handle = handle
        self.desc = desc

    @property
    def D(self) -> int:
        return self.desc.n_kv_heads * self.desc.head_dim

    def __del__(self):
        if getattr(self, "handle", None):
            try:
                _lib.lr_cache_destroy(self.handle)
            except Exception:
                pass
            self.handle = None


def _groups(desc) -> int:
    return desc.latent_groups if desc.latent_groups > 1 else 1


def _basis_shapes(desc, r):
    """(A shape, B shape) of the bases a caller passes: [D][r], [r][D], or per group."""
    D, g = desc.n_kv_heads * desc.head_dim, _groups(desc)
    if g == 1:
        return (D, r), (r, D)
    return (g, D // g, r), (g, r, D // g)


def lr_cache_create(desc: lr_cache_desc, A_k, B_k, A_v, B_v, stream=None) -> Cache:
    dt = _torch_dtype(desc.dtype)
    ak, bk = _basis_shapes(desc, desc.rank_k)
    av, bv = _basis_shapes(desc, desc.rank_v)
    out = ctypes.c_void_p()
    _check(_lib.lr_cache_create(ctypes.byref(desc),
                                _ptr(A_k, dt, ak, "A_k", True), _ptr(B_k, dt, bk, "B_k"),
                                _ptr(A_v, dt, av, "A_v", True), _ptr(B_v, dt, bv, "B_v"),
                                _stream(stream), ctypes.byref(out)), "lr_cache_create")
    return Cache(out, desc)


def lr_cache_destroy(cache: Cache) -> None:
    if cache.handle:
        _check(_lib.lr_cache_destroy(cache.handle), "lr_cache_destroy")
        cache.handle = None


def lr_kv_append(cache: Cache, k, v, stream=None) -> None:
    d, dt = cache.desc, _torch_dtype(cache.desc.dtype)
    _check(_lib.lr_kv_append(cache.handle, _ptr(k, dt, (d.batch, cache.D), "k"),
                             _ptr(v, dt, (d.batch, cache.D), "v"), _stream(stream)), "lr_kv_append")


def lr_kv_append_rows(cache: Cache, k, v, pos, max_len: int, stream=None) -> None:
    """pos: int32 CUDA tensor [batch], the history slot of each row's token."""
    import torch
    d, dt = cache.desc, _torch_dtype(cache.desc.dtype)
    _check(_lib.lr_kv_append_rows(cache.handle, _ptr(k, dt, (d.batch, cache.D), "k"),
                                  _ptr(v, dt, (d.batch, cache.D), "v"),
                                  _ptr(pos, torch.int32, (d.batch,), "pos"), int(max_len), _stream(stream)),
           "lr_kv_append_rows")


def lr_kv_prefill(cache: Cache, k, v, stream=None) -> None:
    """k, v: CUDA tensors [batch][n][D] in the cache dtype."""
    d, dt = cache.desc, _torch_dtype(cache.desc.dtype)
    n = k.shape[1] if k.dim() == 3 else -1
    _check(_lib.lr_kv_prefill(cache.handle, _ptr(k, dt, (d.batch, n, cache.D), "k"),
                              _ptr(v, dt, (d.batch, n, cache.D), "v"), n, _stream(stream)), "lr_kv_prefill")


def lr_kv_append_latent(cache: Cache, z_k, z_v, stream=None) -> None:
    import torch
    d = cache.desc
    g = _groups(d)
    n = z_k.shape[1] if z_k.dim() == 3 else -1
    _check(_lib.lr_kv_append_latent(cache.handle,
                                    _ptr(z_k, torch.float32, (d.batch, n, g * d.rank_k), "z_k"),
                                    _ptr(z_v, torch.float32, (d.batch, n, g * d.rank_v), "z_v"),
                                    n, _stream(stream)), "lr_kv_append_latent")


def lr_attn_decode(cache: Cache, q, out, lse=None, stream=None) -> None:
    import torch
    d, dt = cache.desc, _torch_dtype(cache.desc.dtype)
    shp = (d.batch, d.n_q_heads, d.head_dim)
    _check(_lib.lr_attn_decode(cache.handle, _ptr(q, dt, shp, "q"), _ptr(out, dt, shp, "out"),
                               _ptr(lse, torch.float32, (d.batch, d.n_q_heads), "lse", True),
                               _stream(stream)), "lr_attn_decode")


def lr_attn_decode_varlen(cache: Cache, q, out, row_len, lse=None, stream=None) -> None:
    """row_len: int32 CUDA tensor [batch], tokens of history each row attends to."""
    import torch
    d, dt = cache.desc, _torch_dtype(cache.desc.dtype)
    shp = (d.batch, d.n_q_heads, d.head_dim)
    _check(_lib.lr_attn_decode_varlen(cache.handle, _ptr(q, dt, shp, "q"), _ptr(out, dt, shp, "out"),
                                      _ptr(lse, torch.float32, (d.batch, d.n_q_heads), "lse", True),
                                      _ptr(row_len, torch.int32, (d.batch,), "row_len"),
                                      _stream(stream)), "lr_attn_decode_varlen")


def lr_attn_decode_partial(cache: Cache, q, part_o, part_ml, stream=None) -> None:
    """part_o: fp32 CUDA tensor [batch][Hq][r_v], part_ml: [batch][Hq][2]."""
    import torch
    d, dt = cache.desc, _torch_dtype(cache.desc.dtype)
    rv = _groups(d) * d.rank_v
    _check(_lib.lr_attn_decode_partial(cache.handle, _ptr(q, dt, (d.batch, d.n_q_heads, d.head_dim), "q"),
                                       _ptr(part_o, torch.float32, (d.batch, d.n_q_heads, rv), "part_o"),
                                       _ptr(part_ml, torch.float32, (d.batch, d.n_q_heads, 2), "part_ml"),
                                       _stream(stream)), "lr_attn_decode_partial")


def lr_merge_partials(cache: Cache, part_o, part_ml, out, lse=None, stream=None) -> None:
    """part_o: fp32 [n][batch][Hq][r_v], part_ml: [n][batch][Hq][2] (n shards' partials)."""
    import torch
    d, dt = cache.desc, _torch_dtype(cache.desc.dtype)
    rv = _groups(d) * d.rank_v
    n = part_o.shape[0]
    _check(_lib.lr_merge_partials(cache.handle, int(n),
                                  _ptr(part_o, torch.float32, (n, d.batch, d.n_q_heads, rv), "part_o"),
                                  _ptr(part_ml, torch.float32, (n, d.batch, d.n_q_heads, 2), "part_ml"),
                                  _ptr(out, dt, (d.batch, d.n_q_heads, d.head_dim), "out"),
                                  _ptr(lse, torch.float32, (d.batch, d.n_q_heads), "lse", True),
                                  _stream(stream)), "lr_merge_partials")


def lr_decode_step(cache: Cache, k, v, q, out, lse=None, stream=None) -> None:
    import torch
    d, dt = cache.desc, _torch_dtype(cache.desc.dtype)
    shp = (d.batch, d.n_q_heads, d.head_dim)
    _check(_lib.lr_decode_step(cache.handle, _ptr(k, dt, (d.batch, cache.D), "k"),
                               _ptr(v, dt, (d.batch, cache.D), "v"), _ptr(q, dt, shp, "q"),
                               _ptr(out, dt, shp, "out"),
                               _ptr(lse, torch.float32, (d.batch, d.n_q_heads), "lse", True),
                               _stream(stream)), "lr_decode_step")


def lr_basis_sync(cache: Cache, R_k=None, R_v=None, B_k_new=None, B_v_new=None, A_k_new=None,
                  A_v_new=None, stream=None) -> None:
    import torch
    d, dt = cache.desc, _torch_dtype(cache.desc.dtype)
    g = _groups(d)
    ak, bk = _basis_shapes(d, d.rank_k)
    av, bv = _basis_shapes(d, d.rank_v)
    rk = (d.rank_k, d.rank_k) if g == 1 else (g, d.rank_k, d.rank_k)
    rv = (d.rank_v, d.rank_v) if g == 1 else (g, d.rank_v, d.rank_v)
    _check(_lib.lr_basis_sync(cache.handle,
                              _ptr(R_k, torch.float32, rk, "R_k", True),
                              _ptr(R_v, torch.float32, rv, "R_v", True),
                              _ptr(B_k_new, dt, bk, "B_k_new", True),
                              _ptr(B_v_new, dt, bv, "B_v_new", True),
                              _ptr(A_k_new, dt, ak, "A_k_new", True),
                              _ptr(A_v_new, dt, av, "A_v_new", True),
                              _stream(stream)), "lr_basis_sync")


def lr_basis_update(cache: Cache, side: int, blk, gram, R_out, B_new=None, A_new=None, stream=None) -> None:
    """Block-incremental SVD update of the keys' (side 0) or values' (side 1) basis from the
    block blk [n][D] (cache dtype): gram [r][r] fp32 in S, out S'; R_out [r][r] fp32 the
    history sync; B_new [r][D], A_new [D][r] (cache dtype) the new basis, or None."""
    import torch
    d, dt = cache.desc, _torch_dtype(cache.desc.dtype)
    r = d.rank_k if side == 0 else d.rank_v
    D = d.n_kv_heads * d.head_dim
    if blk is None or blk.dim() != 2 or blk.shape[1] != D:
        raise ValueError(f"blk must be [n][{D}]")
    _check(_lib.lr_basis_update(cache.handle, int(side), _ptr(blk, dt, None, "blk"), int(blk.shape[0]),
                                _ptr(gram, torch.float32, (r, r), "gram"),
                                _ptr(R_out, torch.float32, (r, r), "R_out"),
                                _ptr(B_new, dt, (r, D), "B_new", True),
                                _ptr(A_new, dt, (D, r), "A_new", True),
                                _stream(stream)), "lr_basis_update")


LR_NOALLOC_SCRATCH_BYTES = 8 * 1024 * 1024


def _addr(x) -> ctypes.c_void_p:
    """Device address of a CUDA tensor, or an address given as an int."""
    return ctypes.c_void_p(x.data_ptr() if hasattr(x, "data_ptr") else int(x))


def lr_attn_decode_noalloc(desc: lr_cache_desc, length: int, z_k, z_v, B_k, B_v,
                           q, out, lse=None, stream=None) -> None:
    """Decode without device allocation (working memory in the library's static device
    array).  z_k, z_v, B_k, B_v: caller-owned device buffers in the cache layout (CUDA
    tensors or device addresses as ints); q, out (and lse) are CUDA tensors."""
    import torch
    dt = _torch_dtype(desc.dtype)
    shp = (desc.batch, desc.n_q_heads, desc.head_dim)
    _check(_lib.lr_attn_decode_noalloc(ctypes.byref(desc), int(length), _addr(z_k),
                                       _addr(z_v), _addr(B_k), _addr(B_v),
                                       _ptr(q, dt, shp, "q"), _ptr(out, dt, shp, "out"),
                                       _ptr(lse, torch.float32, (desc.batch, desc.n_q_heads), "lse", True),
                                       _stream(stream)), "lr_attn_decode_noalloc")


def lr_cache_get_len(cache: Cache):
    a, b, c = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(_lib.lr_cache_get_len(cache.handle, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
           "lr_cache_get_len")
    return a.value, b.value, c.value


def lr_cache_truncate(cache: Cache, length: int) -> None:
    _check(_lib.lr_cache_truncate(cache.handle, int(length)), "lr_cache_truncate")


def lr_cache_view_get(cache: Cache) -> lr_cache_view:
    v = lr_cache_view()
    _check(_lib.lr_cache_view_get(cache.handle, ctypes.byref(v)), "lr_cache_view_get")
    return v


def lr_cache_set_block_table(cache: Cache, table, stream=None) -> None:
    """table: host array-like of int32, [batch][capacity / 128], the page of each 128-token
    span of each sequence of a paged cache."""
    import numpy as np
    d = cache.desc
    t = np.ascontiguousarray(np.asarray(table), dtype=np.int32)
    if t.shape != (d.batch, d.capacity // 128):
        raise ValueError(f"table must be [{d.batch}][{d.capacity // 128}], got {t.shape}")
    _check(_lib.lr_cache_set_block_table(cache.handle, t.ctypes.data_as(ctypes.c_void_p), _stream(stream)),
           "lr_cache_set_block_table")


def lr_cache_set_block_table_device(cache: Cache, table, stream=None) -> None:
    """table: int32 CUDA tensor [batch][capacity / 128] (entries are not checked; the kernels
    clamp them into the pool)."""
    import torch
    d = cache.desc
    _check(_lib.lr_cache_set_block_table_device(cache.handle, _ptr(table, torch.int32, (d.batch, d.capacity // 128),
                                                                   "table"), _stream(stream)),
           "lr_cache_set_block_table_device")


def lr_cache_set_path(cache: Cache, path: int = LR_PATH_AUTO, n_splits: int = 0) -> None:
    _check(_lib.lr_cache_set_path(cache.handle, int(path), int(n_splits)), "lr_cache_set_path")


def lr_cache_plan(cache: Cache) -> lr_plan:
    p = lr_plan()
    _check(_lib.lr_cache_plan(cache.handle, ctypes.byref(p)), "lr_cache_plan")
    return p


def lr_plan_decode(desc: lr_cache_desc, length: int, num_sms: int, path: int = LR_PATH_AUTO,
                   n_splits: int = 0) -> lr_plan:
    p = lr_plan()
    _check(_lib.lr_plan_decode(ctypes.byref(desc), int(length), int(num_sms), int(path),
                               int(n_splits), ctypes.byref(p)), "lr_plan_decode")
    return p


def lr_cache_set_kernel_events(cache: Cache, ev_start=None, ev_stop=None) -> None:
    """ev_start / ev_stop: torch.cuda.Event objects (already recorded once), or None."""
    a = ctypes.c_void_p(ev_start.cuda_event) if ev_start is not None else None
    b = ctypes.c_void_p(ev_stop.cuda_event) if ev_stop is not None else None
    _check(_lib.lr_cache_set_kernel_events(cache.handle, a, b), "lr_cache_set_kernel_events")


LR_TRACE_SLOTS = 72


def lr_cache_set_trace(cache: Cache, buf=None) -> None:
    """buf: int64 CUDA tensor with >= LR_TRACE_SLOTS * batch * max-splits elements, or None."""
    if buf is None:
        _check(_lib.lr_cache_set_trace(cache.handle, None, 0), "lr_cache_set_trace")
        return
    _check(_lib.lr_cache_set_trace(cache.handle, _ptr(buf, None, None, "trace"), buf.numel()),
           "lr_cache_set_trace")


def lr_abi_struct_sizes():
    a, b, c = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _lib.lr_abi_struct_sizes(ctypes.byref(a), ctypes.byref(b), ctypes.byref(c))
    return a.value, b.value, c.value


LR_FAULT_ALLOC, LR_FAULT_LAUNCH = 0, 1


def lr_cache_set_wait_limit(cache: Cache, ns: int = 0) -> None:
    _check(_lib.lr_cache_set_wait_limit(cache.handle, int(ns)), "lr_cache_set_wait_limit")


def lr_debug_inject_fault(kind: int, after: int) -> None:
    _check(_lib.lr_debug_inject_fault(int(kind), int(after)), "lr_debug_inject_fault")


def lr_device_error(cache: Cache) -> int:
    code = ctypes.c_int32()
    _check(_lib.lr_device_error(cache.handle, ctypes.byref(code)), "lr_device_error")
    return code.value


def raw_status(fn_name: str, *args) -> int:
    """Call a C entry point with raw ctypes arguments and return its status (tests)."""
    return int(getattr(_lib, fn_name)(*args))


class _DeviceArray:
    """Describes raw cache storage through __cuda_array_interface__ (no copy)."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 2, "strides": None}


def copy_view(ptr: int, shape, typestr: str):
    """Clone cache storage at device address `ptr` into a new CUDA tensor.
    typestr: '<f4', '<i2' (bf16 bit patterns), '<i4' (codes / params), ..."""
    import torch
    return torch.as_tensor(_DeviceArray(ptr, shape, typestr), device="cuda").clone()
