"""Paged caches (page_tokens = 128, lr_cache_set_block_table): the latents of every sequence
live in 128-token pages of one pool, in whatever order the block table gives.  Paging is a
storage layout only, so every result must be BIT-IDENTICAL to that of a contiguous cache
holding the same latents (same kernels, same per-token arithmetic, same splits), and within
the parity bars of the oracle.  Covered: every decode path (tensor-core bf16, int4 in rank
space, int4 keys before RoPE, CUDA cores fp32 / bf16 / int4), fills, prefills that start
inside a page and cross into the next, fused decode steps, variable-length rows, the basis
sync (tensor-core and CUDA-core), pages shared by several sequences, a table change after
the fill, and the refusals."""
import dataclasses

import numpy as np
import pytest

import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _create(lib, p, cap, paged, n_pages=0, table=None):
    import torch
    d = H.desc_for(lib, p, cap)
    if paged:
        d.page_tokens, d.n_pages = 128, n_pages
    c = lib.lr_cache_create(d, H.to_dev(p, p.A_k), H.to_dev(p, p.B_k), H.to_dev(p, p.A_v), H.to_dev(p, p.B_v))
    if table is not None:
        lib.lr_cache_set_block_table(c, table)
    # two fills: the second starts inside a page (and, for int4 values, inside an 8-token word)
    cut = min(p.hist_len, 301)
    for s, e in ((0, cut), (cut, p.hist_len)):
        if e > s:
            lib.lr_kv_append_latent(c, torch.from_numpy(np.ascontiguousarray(p.z_k[:, s:e])).cuda(),
                                    torch.from_numpy(np.ascontiguousarray(p.z_v[:, s:e])).cuda())
    return c


def _shuffled_table(p, cap, spare, seed):
    pps = cap // 128
    n_pages = p.batch * pps + spare
    perm = np.random.default_rng(seed).permutation(n_pages)
    return n_pages, perm[:p.batch * pps].reshape(p.batch, pps).astype(np.int32)


def _decode(lib, p, c, q, row_len=None):
    import torch
    qd = H.to_dev(p, q)
    out = torch.empty_like(qd)
    lse = torch.empty((p.batch, p.n_q_heads), dtype=torch.float32, device="cuda")
    if row_len is None:
        lib.lr_attn_decode(c, qd, out, lse)
    else:
        lib.lr_attn_decode_varlen(c, qd, out, torch.tensor(row_len, dtype=torch.int32, device="cuda"), lse)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy()


def _same(a, b, tag):
    for x, y in zip(a, b):
        assert np.array_equal(x, y), f"{tag}: paged and contiguous differ (max {np.max(np.abs(x - y)):.3e})"


def _problem(kind):
    if kind == "tiny":
        base = synth.make_tiny(length=250)
        nb = 3
        f = np.array([1.0, -0.5, 2.0], np.float32)[:, None, None]    # distinct rows
        return dataclasses.replace(base, batch=nb, z_k=np.repeat(base.z_k, nb, 0) * f,
                                   z_v=np.repeat(base.z_v, nb, 0), q=np.repeat(base.q, nb, 0))
    if kind == "qwen32k":
        return synth.small_variant("qwen32k", layer=0, batch=3, length=659)
    if kind == "qwen16k":
        return synth.small_variant("qwen16k", batch=3, length=1003)
    return synth.small_variant(kind, batch=3, length=1003)


CASES = [("tiny", None), ("qwen4k", None), ("qwen4k", "simt"), ("qwen16k", None), ("qwen16k", "simt"),
         ("qwen32k", None)]


@pytest.mark.parametrize("kind,path", CASES)
def test_paged_equals_contiguous_and_matches_oracle(lib, kind, path):
    import torch
    p = _problem(kind)
    cap = (p.hist_len + 40 + 127) // 128 * 128 + 128       # room for a prefill across a page edge
    n_pages, table = _shuffled_table(p, cap, spare=5, seed=len(kind) + (path is not None))
    c0 = _create(lib, p, cap, False)
    c1 = _create(lib, p, cap, True, n_pages, table)
    if path == "simt":
        for c in (c0, c1):
            lib.lr_cache_set_path(c, lib.LR_PATH_SIMT)
    q = p.store(H.stored_value(p, p.q) * H.sharp_factor(p))
    a, b = _decode(lib, p, c0, q), _decode(lib, p, c1, q)
    _same(a, b, f"{kind}/{path} decode")
    # against the oracle
    ref, ref_lse = H.oracle_decode(p, q)
    tc_int4 = lib.lr_cache_plan(c1).path == lib.LR_PATH_TC and p.quant_bits == 4
    H.compare(p, b[0].astype(np.float64), ref, b[1].astype(np.float64), ref_lse, tag=f"paged {kind}/{path}",
              lse_tol=H.decode_lse_bound(p, q) if tc_int4 else None)
    # variable-length rows (a row ending on a page edge, one past it, the full history)
    lens = [128, 129, p.hist_len][:p.batch]
    _same(_decode(lib, p, c0, q, lens), _decode(lib, p, c1, q, lens), f"{kind}/{path} varlen")
    # a prefill of exact tokens that starts inside a page and crosses into the next one
    if not p.rope:
        rng = np.random.default_rng(7)
        n = 40
        kx = p.store(rng.standard_normal((p.batch, n, p.kv_dim)) * 0.5)
        vx = p.store(rng.standard_normal((p.batch, n, p.kv_dim)) * 0.5)
        for c in (c0, c1):
            lib.lr_kv_prefill(c, H.to_dev(p, kx), H.to_dev(p, vx))
        _same(_decode(lib, p, c0, q), _decode(lib, p, c1, q), f"{kind}/{path} after prefill")
        # fused decode steps (append + query projection + decode)
        for step in range(3):
            k1 = p.store(rng.standard_normal((p.batch, p.kv_dim)) * 0.5)
            v1 = p.store(rng.standard_normal((p.batch, p.kv_dim)) * 0.5)
            outs = []
            for c in (c0, c1):
                out = torch.empty((p.batch, p.n_q_heads, p.head_dim), dtype=H.to_dev(p, q).dtype, device="cuda")
                lib.lr_decode_step(c, H.to_dev(p, k1), H.to_dev(p, v1), H.to_dev(p, q), out)
                torch.cuda.synchronize()
                outs.append(out.float().cpu().numpy())
            assert np.array_equal(outs[0], outs[1]), f"{kind}/{path} step {step}"
    for c in (c0, c1):
        lib.lr_cache_destroy(c)


@pytest.mark.parametrize("path", [None, "simt"])
def test_paged_basis_sync_rotates_every_page_once(lib, path):
    """The sync rotates the whole pool (each page once): the decode after it equals the
    contiguous cache's, bit for bit, on the tensor-core sync and on the CUDA-core sync."""
    import torch
    p = synth.small_variant("hybrid", hist_len=700, batch=2, window=0, win_len=0)
    cap = 768
    n_pages, table = _shuffled_table(p, cap, spare=3, seed=11)
    c0, c1 = _create(lib, p, cap, False), _create(lib, p, cap, True, n_pages, table)
    if path == "simt":
        for c in (c0, c1):
            lib.lr_cache_set_path(c, lib.LR_PATH_SIMT)
    Rk = synth.sync_rotation(0, 2, p.rank_k, "k")
    Rv = synth.sync_rotation(0, 2, p.rank_v, "v")
    Bk_new = p.store(Rk.T @ H.stored_value(p, p.B_k))
    Bv_new = p.store(Rv.T @ H.stored_value(p, p.B_v))
    for c in (c0, c1):
        lib.lr_basis_sync(c, torch.from_numpy(Rk.astype(np.float32)).cuda(),
                          torch.from_numpy(Rv.astype(np.float32)).cuda(), H.to_dev(p, Bk_new), H.to_dev(p, Bv_new),
                          None, None)
    q = p.store(H.stored_value(p, p.q) * H.sharp_factor(p))
    _same(_decode(lib, p, c0, q), _decode(lib, p, c1, q), f"sync {path}")
    for c in (c0, c1):
        lib.lr_cache_destroy(c)


@pytest.mark.parametrize("kind", ["qwen4k", "qwen16k"])
def test_shared_pages(lib, kind):
    """Every sequence maps the same pages (a common prefix): a pool of capacity / 128 pages
    serves the whole batch and each row's decode equals the contiguous cache that holds the
    prefix once per row."""
    base = synth.small_variant(kind, batch=1, length=600)
    nb = 3
    p = dataclasses.replace(base, batch=nb, z_k=np.repeat(base.z_k, nb, 0), z_v=np.repeat(base.z_v, nb, 0),
                            q=synth.small_variant(kind, batch=nb, length=1).q)
    cap = 640
    pps = cap // 128
    table = np.tile(np.arange(pps, dtype=np.int32)[::-1], (nb, 1))
    c0, c1 = _create(lib, p, cap, False), _create(lib, p, cap, True, pps, table)
    q = p.store(H.stored_value(p, p.q) * H.sharp_factor(p))
    _same(_decode(lib, p, c0, q), _decode(lib, p, c1, q), f"shared {kind}")
    assert lib.lr_cache_view_get(c1).n_pages == pps
    for c in (c0, c1):
        lib.lr_cache_destroy(c)


def test_table_change_after_fill_is_honoured(lib):
    """Swapping two sequences' table rows swaps which latents they attend to: with the
    queries swapped too, the outputs are the old outputs swapped, bit for bit."""
    p = synth.small_variant("qwen4k", batch=2, length=900)
    cap = 1024
    n_pages, table = _shuffled_table(p, cap, spare=0, seed=5)
    c = _create(lib, p, cap, True, n_pages, table)
    q = p.store(H.stored_value(p, p.q) * H.sharp_factor(p))
    out0, lse0 = _decode(lib, p, c, q)
    lib.lr_cache_set_block_table(c, table[::-1].copy())
    out1, lse1 = _decode(lib, p, c, q[::-1].copy())
    assert np.array_equal(out1, out0[::-1]) and np.array_equal(lse1, lse0[::-1])
    lib.lr_cache_destroy(c)


def test_block_table_refusals(lib):
    p = synth.small_variant("qwen4k", batch=2, length=300)
    c0 = _create(lib, p, 384, False)
    with pytest.raises(lib.LRError) as e:
        lib.lr_cache_set_block_table(c0, np.zeros((2, 3), np.int32))
    assert e.value.status == lib.LR_ERR_UNSUPPORTED
    n_pages, table = _shuffled_table(p, 384, spare=1, seed=3)
    c1 = _create(lib, p, 384, True, n_pages, table)
    q = p.q
    before = _decode(lib, p, c1, q)
    for bad in (n_pages, -1):
        t = table.copy()
        t[1, 2] = bad
        with pytest.raises(lib.LRError) as e:
            lib.lr_cache_set_block_table(c1, t)
        assert e.value.status == lib.LR_ERR_INVALID_ARG
    _same(before, _decode(lib, p, c1, q), "after refused tables")
    _same(before, _decode(lib, p, c0, q), "paged against contiguous")
    for c in (c0, c1):
        lib.lr_cache_destroy(c)


def test_device_table_matches_host_table_and_clamps(lib):
    """A block table set from device memory decodes like the same table set from the host;
    entries outside the pool are clamped into it by the kernels (no error, no access outside
    the storage): the result equals the host table with the clamped entries."""
    import torch
    p = synth.small_variant("qwen16k", batch=3, length=700)
    cap = 768
    n_pages, table = _shuffled_table(p, cap, spare=2, seed=9)
    c = _create(lib, p, cap, True, n_pages, table)
    q = p.store(H.stored_value(p, p.q) * H.sharp_factor(p))
    host = _decode(lib, p, c, q)
    lib.lr_cache_set_block_table_device(c, torch.from_numpy(table).cuda())
    _same(host, _decode(lib, p, c, q), "device table")
    bad = table.copy()
    bad[1, 0], bad[2, 3] = -5, n_pages + 3
    lib.lr_cache_set_block_table_device(c, torch.from_numpy(bad).cuda())
    got = _decode(lib, p, c, q)
    assert lib.lr_device_error(c) == 0
    lib.lr_cache_set_block_table(c, np.clip(bad, 0, n_pages - 1))
    _same(got, _decode(lib, p, c, q), "clamped entries")
    lib.lr_cache_destroy(c)


def test_device_table_update_inside_a_cuda_graph(lib):
    """The device-side table update is capturable: a graph of (table update, decode) replayed
    after the table's device buffer changes decodes with the new table."""
    import torch
    p = synth.small_variant("qwen4k", batch=2, length=600)
    cap = 640
    n_pages, table = _shuffled_table(p, cap, spare=0, seed=2)
    c = _create(lib, p, cap, True, n_pages, table)
    q = p.store(H.stored_value(p, p.q) * H.sharp_factor(p))
    qd = H.to_dev(p, q)
    out = torch.empty_like(qd)
    tdev = torch.from_numpy(table).cuda()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        lib.lr_cache_set_block_table_device(c, tdev, stream=s)
        lib.lr_attn_decode(c, qd, out, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lib.lr_cache_set_block_table_device(c, tdev)
        lib.lr_attn_decode(c, qd, out)
    torch.cuda.synchronize()
    for tab in (table[::-1].copy(), table):   # swapped rows, then the original
        tdev.copy_(torch.from_numpy(tab))
        g.replay()
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        lib.lr_cache_set_block_table(c, tab)
        want, _ = _decode(lib, p, c, q)
        assert np.array_equal(got, want)
    del g
    lib.lr_cache_destroy(c)
