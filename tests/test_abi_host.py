"""CPU-only checks of the C ABI: the library loads and exports every symbol the header
declares, struct layouts agree with the binding, and the host-side logic (validation,
planning, status names) behaves without touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lr_kv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(lr_[a-z0-9_]+)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary_calls():
    names = declared_functions()
    for must in ("lr_cache_create", "lr_cache_destroy", "lr_kv_append", "lr_kv_append_latent",
                 "lr_attn_decode", "lr_basis_sync"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    so = ctypes.CDLL(lib.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(so, n)]
    assert not missing, missing


def test_binding_keeps_every_declared_name(lib):
    """The Python binding exposes each C call under its own name."""
    missing = [n for n in declared_functions() if not callable(getattr(lib, n, None))]
    assert not missing, missing


def test_struct_sizes_match_binding(lib):
    assert lib.lr_abi_struct_sizes() == (ctypes.sizeof(lib.lr_cache_desc),
                                         ctypes.sizeof(lib.lr_cache_view),
                                         ctypes.sizeof(lib.lr_plan))


def test_status_strings(lib):
    for code, name in [(0, "LR_OK"), (1, "LR_ERR_INVALID_ARG"), (2, "LR_ERR_UNSUPPORTED"),
                       (3, "LR_ERR_CAPACITY"), (4, "LR_ERR_CUDA"), (5, "LR_ERR_OOM"),
                       (6, "LR_ERR_TIMEOUT"), (99, "LR_ERR_UNKNOWN")]:
        assert lib.lr_status_string(code) == name


def _qwen(lib, **kw):
    base = dict(batch=16, n_q_heads=28, n_kv_heads=4, head_dim=128, rank_k=256, rank_v=256,
                capacity=4096)
    base.update(kw)
    return lib.make_desc(**base)


@pytest.mark.parametrize("field,value,status", [
    ("n_q_heads", 27, 1), ("head_dim", 127, 1), ("rank_k", 250, 1), ("rank_v", 1024, 1),
    ("quant_bits", 3, 1), ("quant_group", 64, 2), ("dtype", 7, 1), ("window", 5000, 1),
    ("batch", 0, 1), ("capacity", 0, 1)])
def test_invalid_descriptions_rejected_before_device(lib, field, value, status):
    kw = {field: value}
    if field == "quant_group":
        kw["quant_bits"] = 4
    d = _qwen(lib, **kw)
    out = ctypes.c_void_p()
    st = lib.raw_status("lr_cache_create", ctypes.byref(d), None, ctypes.c_void_p(1), None,
                        ctypes.c_void_p(1), None, ctypes.byref(out))
    assert st == status and not out.value


def test_rope_with_window_is_unsupported(lib):
    d = _qwen(lib, rope_in_kernel=1, window=128)
    with pytest.raises(lib.LRError) as e:
        lib.lr_plan_decode(d, 1000, 148)
    assert e.value.status == lib.LR_ERR_UNSUPPORTED


def test_reserved_fields_must_be_zero(lib):
    for i in range(2):
        d = _qwen(lib)
        d.reserved[i] = 1
        with pytest.raises(lib.LRError):
            lib.lr_plan_decode(d, 10, 148)


@pytest.mark.parametrize("page_tokens, n_pages, capacity, window, status", [
    (128, 0, 4096, 0, 0),        # default pool: batch * capacity / 128 pages
    (128, 5, 4096, 0, 0),        # a pool smaller than the table (pages shared or unused)
    (64, 0, 4096, 0, 1),         # pages are 128 tokens
    (0, 8, 4096, 0, 1),          # a pool size without paging
    (128, -1, 4096, 0, 1),
    (128, 1 << 23, 4096, 0, 1),  # above the pool limit
    (128, 0, 4000, 0, 2),        # capacity not a whole number of pages
    (128, 0, 4096, 128, 2),      # no exact window in a paged cache
])
def test_paged_desc_validation(lib, page_tokens, n_pages, capacity, window, status):
    d = _qwen(lib, capacity=capacity, window=window)
    d.page_tokens, d.n_pages = page_tokens, n_pages
    if status == 0:
        lib.lr_plan_decode(d, 100, 148)
    else:
        with pytest.raises(lib.LRError) as e:
            lib.lr_plan_decode(d, 100, 148)
        assert e.value.status == status


def test_noalloc_refuses_paged_desc_before_any_device_call(lib):
    d = _qwen(lib)
    d.page_tokens = 128
    dummy = ctypes.c_void_p(256)
    st = lib.raw_status("lr_attn_decode_noalloc", ctypes.byref(d), 100, dummy, dummy, dummy, dummy, dummy,
                        dummy, None, None)
    assert st == lib.LR_ERR_UNSUPPORTED


def test_null_arguments(lib):
    assert lib.raw_status("lr_kv_append", None, None, None, None) == lib.LR_ERR_INVALID_ARG
    assert lib.raw_status("lr_kv_append_rows", None, None, None, None, 0, None) == lib.LR_ERR_INVALID_ARG
    assert lib.raw_status("lr_attn_decode", None, None, None, None, None) == lib.LR_ERR_INVALID_ARG
    assert lib.raw_status("lr_cache_destroy", None) == lib.LR_OK


@pytest.mark.parametrize("length", [1, 17, 128, 1000, 4096, 4095])
@pytest.mark.parametrize("batch", [1, 8, 16])
@pytest.mark.parametrize("path", [1, 0])
def test_plan_covers_history_exactly(lib, length, batch, path):
    d = _qwen(lib, batch=batch)
    p = lib.lr_plan_decode(d, length, 148, path)
    assert p.split_tokens % p.tile_tokens == 0
    assert (p.n_splits - 1) * p.split_tokens < length <= p.n_splits * p.split_tokens
    assert p.ctas == p.n_splits * batch
    assert p.n_splits * batch <= max(2 * 148 + batch, batch)


@pytest.mark.parametrize("n_kv_heads, pairs", [(4, 2), (2, 1)])
@pytest.mark.parametrize("rank_k", [128, 256, 448])
def test_plan_keys_before_rope_int4_on_kv_head_pairs(lib, n_kv_heads, pairs, rank_k):
    """int4 keys before RoPE take the tensor-core path with one CTA per pair of KV heads,
    within one wave of 148 SMs."""
    d = _qwen(lib, n_q_heads=7 * n_kv_heads, n_kv_heads=n_kv_heads, rank_k=rank_k, rank_v=448,
              quant_bits=4, rope_in_kernel=1, capacity=32768)
    p = lib.lr_plan_decode(d, 32768, 148)
    assert p.path == lib.LR_PATH_TC
    assert p.ctas == p.n_splits * d.batch * pairs
    assert p.ctas <= 148
    assert (p.n_splits - 1) * p.split_tokens < 32768 <= p.n_splits * p.split_tokens


@pytest.mark.parametrize("shape", [dict(n_q_heads=16, n_kv_heads=4), dict(n_q_heads=7, n_kv_heads=1),
                                   dict(n_q_heads=21, n_kv_heads=3), dict(n_q_heads=64, n_kv_heads=4)])
def test_plan_keys_before_rope_on_tensor_cores_for_head_groups_up_to_16(lib, shape):
    """The tensor-core keys-before-RoPE variant takes d = 128 with up to 16 query heads per
    KV head (the score MMA's N), one CTA per pair of KV heads, or per KV head when their
    number is odd."""
    d = _qwen(lib, quant_bits=4, rope_in_kernel=1, **shape)
    p = lib.lr_plan_decode(d, 4096, 148)
    assert p.path == lib.LR_PATH_TC
    per = 2 if shape["n_kv_heads"] % 2 == 0 else 1
    assert p.ctas == p.n_splits * d.batch * (shape["n_kv_heads"] // per)


@pytest.mark.parametrize("shape", [dict(head_dim=64), dict(n_q_heads=20, n_kv_heads=1),
                                   dict(n_q_heads=68, n_kv_heads=2)])
def test_plan_keys_before_rope_other_shapes_use_cuda_cores(lib, shape):
    """Other head dimensions, and more than 16 query heads per KV head, decode on CUDA cores."""
    d = _qwen(lib, quant_bits=4, rope_in_kernel=1, **shape)
    assert lib.lr_plan_decode(d, 4096, 148).path == lib.LR_PATH_SIMT


def test_plan_forced_splits_and_window(lib):
    d = _qwen(lib, capacity=8192)
    p = lib.lr_plan_decode(d, 4096, 148, 1, 7)
    assert p.n_splits == 7 and p.split_tokens * 7 >= 4096
    dw = _qwen(lib, batch=8, n_q_heads=32, n_kv_heads=8, capacity=32768, window=128)
    p = lib.lr_plan_decode(dw, 32768, 148, 1)
    assert p.n_splits * p.split_tokens >= 32768 - 128
    assert (p.n_splits - 1) * p.split_tokens < 32768 - 128


def test_fault_injection_arguments(lib):
    """Arming and disarming the host fault injection is host-only bookkeeping."""
    assert lib.raw_status("lr_debug_inject_fault", 2, 0) == lib.LR_ERR_INVALID_ARG
    assert lib.raw_status("lr_debug_inject_fault", lib.LR_FAULT_ALLOC, -2) == lib.LR_ERR_INVALID_ARG
    for kind in (lib.LR_FAULT_ALLOC, lib.LR_FAULT_LAUNCH):
        assert lib.raw_status("lr_debug_inject_fault", kind, 3) == lib.LR_OK
        assert lib.raw_status("lr_debug_inject_fault", kind, -1) == lib.LR_OK


def test_wait_limit_rejects_bad_arguments(lib):
    assert lib.raw_status("lr_cache_set_wait_limit", None, 10) == lib.LR_ERR_INVALID_ARG


def test_latent_groups_validation_and_plan(lib):
    """Latent groups must divide the KV heads, and the ranks they add up to stay within the
    512 limit; the plan is that of the block-diagonal cache of rank g * r."""
    def status(**kw):
        d = _qwen(lib, **kw)
        return lib.raw_status("lr_plan_decode", ctypes.byref(d), 4096, 148, 0, 0, ctypes.byref(lib.lr_plan()))
    assert status(latent_groups=3) == lib.LR_ERR_INVALID_ARG            # 4 KV heads
    assert status(latent_groups=-1) == lib.LR_ERR_INVALID_ARG
    assert status(latent_groups=4, rank_k=160, rank_v=64) == lib.LR_ERR_INVALID_ARG   # 640 > 512
    assert status(latent_groups=4, rank_k=64, rank_v=64) == lib.LR_OK
    grouped = lib.lr_plan_decode(_qwen(lib, latent_groups=4, rank_k=64, rank_v=64), 4096, 148)
    shared = lib.lr_plan_decode(_qwen(lib, rank_k=256, rank_v=256), 4096, 148)
    assert (grouped.path, grouped.n_splits, grouped.ctas) == (shared.path, shared.n_splits, shared.ctas)
