"""Parity at the benchmark's full sizes, on sampled outputs.

The caches have the shapes the bench times (batch 16 at 4K, 16K and 32K tokens; the
hybrid cache at 32K) and are decoded with the automatic plan (the same path, split count
and launch configuration as the bench's step).  The fp64 oracle then computes a seeded
sample of (sequence, query head) outputs one by one, materialising only the sampled
sequences' latents, and the tolerances of the small-size tests apply to every sample."""
import numpy as np
import pytest

import synth
from oracle import attention
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _sampled_oracle(p: synth.Problem, q: np.ndarray, pairs):
    """Oracle outputs for `pairs` only; returns arrays [B][Hq][d] / [B][Hq] with NaN
    elsewhere."""
    rows = sorted({b for b, _ in pairs})
    qv = H.stored_value(p, q)[rows]
    Zk = np.stack([H.oracle_latents(p, p.z_k[b]) for b in rows])
    Zv = np.stack([H.oracle_latents(p, p.z_v[b]) for b in rows])
    wk = H.stored_value(p, p.win_k[rows]) if p.win_k is not None else None
    wv = H.stored_value(p, p.win_v[rows]) if p.win_v is not None else None
    sub_pairs = [(rows.index(b), j) for b, j in pairs]
    o, l = attention.decode(qv, Zk, Zv, H.stored_value(p, p.B_k), H.stored_value(p, p.B_v), p.n_kv_heads,
                            None, p.rope_theta if p.rope else None, wk, wv, sub_pairs)
    out = np.full((p.batch, p.n_q_heads, p.head_dim), np.nan)
    lse = np.full((p.batch, p.n_q_heads), np.nan)
    for (b, j), (bs, _) in zip(pairs, sub_pairs):
        out[b, j] = o[bs, j]
        lse[b, j] = l[bs, j]
    return out, lse


def _check(lib, p, count=6, seed=0):
    c = H.fill_cache(lib, p)
    plan = lib.lr_cache_plan(c)
    pairs = attention.sample_pairs(p.batch, p.n_q_heads, count, seed)
    f = H.sharp_factor(p)
    for q in (p.q, p.store(H.stored_value(p, p.q) * f)):
        ref, ref_lse = _sampled_oracle(p, q, pairs)
        got, lse = H.gpu_decode(lib, p, c, q)
        lse_tol = None
        if plan.path == lib.LR_PATH_TC and p.quant_bits == 4:
            lse_tol = np.full((p.batch, p.n_q_heads), np.nan)
            bound = H.decode_lse_bound(_rows_only(p, pairs), q[sorted({b for b, _ in pairs})])
            for k, b in enumerate(sorted({b for b, _ in pairs})):
                lse_tol[b] = bound[k]
        H.compare(p, got, ref, lse, ref_lse, pairs=pairs, tag=f"{p.name} T={p.length} path={plan.path}",
                  lse_tol=lse_tol)
    assert lib.lr_device_error(c) == 0
    return plan


def _rows_only(p: synth.Problem, pairs):
    """The problem restricted to the sampled sequences (for the per-sample LSE bound)."""
    import dataclasses
    rows = sorted({b for b, _ in pairs})
    return dataclasses.replace(p, batch=len(rows), z_k=p.z_k[rows], z_v=p.z_v[rows], q=p.q[rows])


def test_fullsize_qwen4k_bf16(lib):
    p = synth.make_qwen("qwen4k", seed=0, batch=16, length=4096, rank=256)
    plan = _check(lib, p)
    assert plan.path == lib.LR_PATH_TC


def test_fullsize_qwen16k_int4(lib):
    p = synth.make_qwen("qwen16k", seed=0, batch=16, length=16384, rank=352, quant_bits=4)
    plan = _check(lib, p)
    assert plan.path == lib.LR_PATH_TC


def test_fullsize_qwen32k_int4_layer(lib):
    # layer 0 of the 28-layer cache, ranks (256, 384), keys stored after RoPE
    p = synth.make_qwen32k_layer(0, seed=0, batch=16, length=32768, rope=False)
    plan = _check(lib, p, count=4)
    assert plan.path == lib.LR_PATH_TC


def test_fullsize_qwen32k_int4_layer_prerope(lib):
    # layer 11 of the 28-layer cache, ranks (448, 256), keys stored before RoPE: the
    # per-tile rebuild and rotation at positions up to 32767
    p = synth.make_qwen32k_layer(11, seed=0, batch=16, length=32768, rope=True)
    plan = _check(lib, p, count=4)
    assert plan.path == lib.LR_PATH_TC


def test_fullsize_hybrid(lib):
    p = synth.make_hybrid(seed=0, batch=8, hist_len=32640)
    plan = _check(lib, p, count=4)
    assert plan.path == lib.LR_PATH_TC


@pytest.mark.parametrize("kind", ["qwen4k", "qwen16k"])
def test_fullsize_paged_equals_contiguous(lib, kind):
    """The bench's layers held in a paged cache (a seeded random permutation of every
    128-token page as block table) decode bit for bit like the contiguous cache, with the
    automatic plan the bench uses."""
    import torch
    if kind == "qwen4k":
        p = synth.make_qwen("qwen4k", seed=0, batch=16, length=4095, rank=256)
        cap = 4096
    else:
        p = synth.make_qwen("qwen16k", seed=0, batch=16, length=16383, rank=352, quant_bits=4)
        cap = 16384
    caches = []
    for paged in (False, True):
        d = H.desc_for(lib, p, cap)
        if paged:
            d.page_tokens = 128
        c = lib.lr_cache_create(d, H.to_dev(p, p.A_k), H.to_dev(p, p.B_k), H.to_dev(p, p.A_v), H.to_dev(p, p.B_v))
        if paged:
            pps = cap // 128
            table = np.random.default_rng(7).permutation(p.batch * pps).astype(np.int32).reshape(p.batch, pps)
            lib.lr_cache_set_block_table(c, table)
        for s0 in range(0, p.hist_len, 2048):
            e0 = min(p.hist_len, s0 + 2048)
            lib.lr_kv_append_latent(c, torch.from_numpy(np.ascontiguousarray(p.z_k[:, s0:e0])).cuda(),
                                    torch.from_numpy(np.ascontiguousarray(p.z_v[:, s0:e0])).cuda())
        caches.append(c)
    q = p.store(H.stored_value(p, p.q) * H.sharp_factor(p))
    (a, la), (b, lb) = (H.gpu_decode(lib, p, c, q) for c in caches)
    assert lib.lr_cache_plan(caches[1]).n_splits == lib.lr_cache_plan(caches[0]).n_splits
    assert np.array_equal(a, b) and np.array_equal(la, lb)
    for c in caches:
        lib.lr_cache_destroy(c)
