"""Per-row appends (lr_kv_append_rows): in a serving batch whose sequences are at different
lengths, each row's new token is projected and stored at that row's own slot, and the batch
is then read with lr_attn_decode_varlen.

The new tokens are one-hot rows scaled by a power of two, so that their latents c * A[i, :]
come out exact in fp32 and in fp64 alike: the oracle then stores the same bf16 values and the
same int4 codes as the device, and any difference is the kernel's.  Checked: the decode of
every row over its own length + 1 against the oracle; a full decode over the whole history,
which shows that no other slot changed (the row whose slot is out of range wrote nothing);
the history length after max_len; bit-identity with lr_kv_append when every row is at the
common length; and the refusals."""
import dataclasses

import numpy as np
import pytest

import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu

L = 300                                    # filled history per row
CAP = 512


def _problem(kind):
    nb = 6
    if kind == "qwen32k":
        return synth.small_variant("qwen32k", layer=0, batch=nb, length=L)
    return synth.small_variant(kind, batch=nb, length=L)


def _cache(lib, p, paged):
    import torch
    d = H.desc_for(lib, p, CAP)
    if paged:
        pps = CAP // 128
        d.page_tokens, d.n_pages = 128, p.batch * pps + 3
    c = lib.lr_cache_create(d, H.to_dev(p, p.A_k), H.to_dev(p, p.B_k), H.to_dev(p, p.A_v), H.to_dev(p, p.B_v))
    if paged:
        perm = np.random.default_rng(5).permutation(d.n_pages)[:p.batch * pps]
        lib.lr_cache_set_block_table(c, perm.reshape(p.batch, pps).astype(np.int32))
    lib.lr_kv_append_latent(c, torch.from_numpy(np.ascontiguousarray(p.z_k)).cuda(),
                            torch.from_numpy(np.ascontiguousarray(p.z_v)).cuda())
    return c


def _one_hot_tokens(p, seed):
    """Scaled one-hot keys and values [B][D] (stored form) and their exact latents."""
    rng = np.random.default_rng(seed)
    D = p.kv_dim
    A_k, A_v = p.to_f64(p.A_k), p.to_f64(p.A_v)
    out = []
    for A, z in ((A_k, p.z_k), (A_v, p.z_v)):
        x = np.zeros((p.batch, D))
        zz = np.zeros((p.batch, A.shape[1]))
        for b in range(p.batch):
            i = int(rng.integers(D))
            c = 2.0 ** np.round(np.log2(np.std(z[b]) / max(np.std(A[i]), 1e-30)))
            x[b, i] = c
            zz[b] = c * A[i]                # one product per coordinate: exact in fp32
        out.append((p.store(x), zz.astype(np.float32)))
    assert np.array_equal(out[0][1].astype(np.float64), p.to_f64(out[0][0]) @ A_k)
    return out


def _with_token(z, pos, znew, length):
    """History latents [B][length][r] after each row b's token is written at pos[b]."""
    B, _, r = z.shape
    zz = np.zeros((B, length, r), np.float32)
    zz[:, :z.shape[1]] = z
    for b in range(B):
        if 0 <= pos[b] < length:
            zz[b, pos[b]] = znew[b]
    return zz


CASES = [("qwen4k", None, False), ("qwen4k", "simt", False), ("qwen16k", None, False),
         ("qwen32k", None, False), ("qwen4k", None, True), ("qwen16k", None, True)]


@pytest.mark.parametrize("kind,path,paged", CASES)
def test_rows_append_at_own_slot_then_varlen_decode(lib, kind, path, paged):
    import torch
    p = _problem(kind)
    p = dataclasses.replace(p, q=p.store(H.stored_value(p, p.q) * H.sharp_factor(p)))
    c = _cache(lib, p, paged)
    if path == "simt":
        lib.lr_cache_set_path(c, lib.LR_PATH_SIMT)
    (kx, zk_new), (vx, zv_new) = _one_hot_tokens(p, seed=11)
    # rows at lengths 1, 127, 128, 200 and L take their next slot; the last row's slot is out
    # of range and writes nothing
    pos = [1, 127, 128, 200, L, CAP]
    lib.lr_kv_append_rows(c, H.to_dev(p, kx), H.to_dev(p, vx),
                          torch.tensor(pos, dtype=torch.int32, device="cuda"), L + 1)
    assert lib.lr_cache_get_len(c) == (L + 1, L + 1, 0)
    zk = _with_token(p.z_k, pos, zk_new, L + 1)
    zv = _with_token(p.z_v, pos, zv_new, L + 1)
    full = dataclasses.replace(p, hist_len=L + 1, z_k=zk, z_v=zv)
    tc_int4 = lib.lr_cache_plan(c).path == lib.LR_PATH_TC and p.quant_bits == 4
    qd = H.to_dev(p, p.q)
    # each row over its own tokens (the last row over its untouched history)
    lens = [n + 1 for n in pos[:-1]] + [L]
    out = torch.empty_like(qd)
    lse = torch.empty((p.batch, p.n_q_heads), dtype=torch.float32, device="cuda")
    lib.lr_attn_decode_varlen(c, qd, out, torch.tensor(lens, dtype=torch.int32, device="cuda"), lse)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().astype(np.float64)
    got_lse = lse.cpu().numpy().astype(np.float64)
    for b, n in enumerate(lens):
        pb = dataclasses.replace(full, batch=1, hist_len=n, z_k=zk[b:b + 1, :n], z_v=zv[b:b + 1, :n],
                                 q=p.q[b:b + 1])
        ref, ref_lse = H.oracle_decode(pb)
        H.compare(pb, got[b:b + 1], ref, got_lse[b:b + 1], ref_lse, tag=f"{kind} row {b} len {n}",
                  lse_tol=H.decode_lse_bound(pb, pb.q) if tc_int4 else None)
    # every row over the whole history: slots other than pos[b] kept their latents (slot L of
    # the rows that did not write it is still zero)
    got, got_lse = H.gpu_decode(lib, full, c)
    ref, ref_lse = H.oracle_decode(full)
    H.compare(full, got, ref, got_lse, ref_lse, tag=f"{kind} full history",
              lse_tol=H.decode_lse_bound(full, full.q) if tc_int4 else None)
    lib.lr_cache_destroy(c)


@pytest.mark.parametrize("kind", ["qwen4k", "qwen16k"])
def test_rows_at_common_length_equal_append(lib, kind):
    """All rows at the common length: bit-identical to lr_kv_append of the same tokens."""
    import torch
    p = _problem(kind)
    rng = np.random.default_rng(3)
    kx = p.store(rng.standard_normal((p.batch, p.kv_dim)) * 0.05)
    vx = p.store(rng.standard_normal((p.batch, p.kv_dim)) * 0.05)
    a, b = _cache(lib, p, False), _cache(lib, p, False)
    lib.lr_kv_append(a, H.to_dev(p, kx), H.to_dev(p, vx))
    lib.lr_kv_append_rows(b, H.to_dev(p, kx), H.to_dev(p, vx),
                          torch.full((p.batch,), L, dtype=torch.int32, device="cuda"), L + 1)
    assert lib.lr_cache_get_len(a) == lib.lr_cache_get_len(b) == (L + 1, L + 1, 0)
    outs = []
    for c in (a, b):
        outs.append(H.gpu_decode(lib, p, c))
    for x, y in zip(*outs):
        assert np.array_equal(x, y)
    lib.lr_cache_destroy(a)
    lib.lr_cache_destroy(b)


def test_rows_refusals(lib):
    import torch
    p = _problem("qwen4k")
    c = _cache(lib, p, False)
    kx = H.to_dev(p, p.store(np.zeros((p.batch, p.kv_dim))))
    pos = torch.zeros((p.batch,), dtype=torch.int32, device="cuda")
    with pytest.raises(lib.LRError) as e:
        lib.lr_kv_append_rows(c, kx, kx, pos, CAP + 1)
    assert e.value.status == lib.LR_ERR_CAPACITY
    with pytest.raises(lib.LRError) as e:
        lib.lr_kv_append_rows(c, kx, kx, pos, -1)
    assert e.value.status == lib.LR_ERR_INVALID_ARG
    assert lib.lr_cache_get_len(c) == (L, L, 0)
    lib.lr_cache_destroy(c)
    w = synth.small_variant("hybrid", hist_len=0, win_len=0, window=8, batch=2)
    cw = lib.lr_cache_create(H.desc_for(lib, w, capacity=64), H.to_dev(w, w.A_k), H.to_dev(w, w.B_k),
                             H.to_dev(w, w.A_v), H.to_dev(w, w.B_v))
    kw = H.to_dev(w, w.store(np.zeros((w.batch, w.kv_dim))))
    with pytest.raises(lib.LRError) as e:
        lib.lr_kv_append_rows(cw, kw, kw, torch.zeros((w.batch,), dtype=torch.int32, device="cuda"), 1)
    assert e.value.status == lib.LR_ERR_UNSUPPORTED
    lib.lr_cache_destroy(cw)


def test_rows_append_and_varlen_decode_in_a_cuda_graph(lib):
    """lr_kv_append_rows and lr_attn_decode_varlen read the positions and the row lengths on
    the device, so one captured graph serves new positions: each replay writes the rows'
    tokens at the positions then in the device tensor and decodes each row over its length,
    checked against the oracle of the cache as the replays have left it."""
    import torch
    p = _problem("qwen4k")
    p = dataclasses.replace(p, q=p.store(H.stored_value(p, p.q) * H.sharp_factor(p)))
    c = _cache(lib, p, False)
    (kx, zk_new), (vx, zv_new) = _one_hot_tokens(p, seed=5)
    kd, vd, qd = H.to_dev(p, kx), H.to_dev(p, vx), H.to_dev(p, p.q)
    pos = torch.zeros((p.batch,), dtype=torch.int32, device="cuda")
    row_len = torch.ones((p.batch,), dtype=torch.int32, device="cuda")
    out = torch.empty_like(qd)
    lse = torch.empty((p.batch, p.n_q_heads), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        lib.lr_kv_append_rows(c, kd, vd, pos, L + 2, stream=s)
        lib.lr_attn_decode_varlen(c, qd, out, row_len, lse, stream=s)
    assert lib.lr_cache_get_len(c) == (L + 2, L + 2, 0)
    zk = _with_token(p.z_k, [CAP] * p.batch, zk_new, L + 2)
    zv = _with_token(p.z_v, [CAP] * p.batch, zv_new, L + 2)
    for rep, positions in enumerate(([5, 128, 299, 300, 301, 0], [127, 3, 300, 301, 64, 200])):
        pos.copy_(torch.tensor(positions, dtype=torch.int32))
        row_len.copy_(torch.tensor([q + 1 for q in positions], dtype=torch.int32))
        g.replay()
        torch.cuda.synchronize()
        for b, q in enumerate(positions):
            zk[b, q] = zk_new[b]
            zv[b, q] = zv_new[b]
        got = out.float().cpu().numpy().astype(np.float64)
        got_lse = lse.cpu().numpy().astype(np.float64)
        full = dataclasses.replace(p, hist_len=L + 2, z_k=zk, z_v=zv)
        for b, q in enumerate(positions):
            n = q + 1
            pb = dataclasses.replace(full, batch=1, hist_len=n, z_k=zk[b:b + 1, :n], z_v=zv[b:b + 1, :n],
                                     q=p.q[b:b + 1])
            ref, ref_lse = H.oracle_decode(pb)
            H.compare(pb, got[b:b + 1], ref, got_lse[b:b + 1], ref_lse, tag=f"graph replay {rep} row {b} len {n}")
    del g
    lib.lr_cache_destroy(c)
