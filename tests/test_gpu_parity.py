"""Parity of the CUDA library (through the C ABI) with the CPU oracle, on seeded synthetic
inputs at sizes the oracle finishes in seconds: several tiles, ragged tails, every
workload family, both decode paths, and the edge cases of the method."""
import dataclasses

import numpy as np
import pytest

import synth
from oracle import attention, iskv, quant
from tests import helpers as H

pytestmark = pytest.mark.gpu


def paths(lr, p=None):
    """Decode paths to check: the fp32 CUDA-core path always, the tcgen05 path where the
    cache supports it."""
    out = [lr.LR_PATH_SIMT]
    if p is not None:
        try:
            lr.lr_plan_decode(H.desc_for(lr, p), max(p.length, 1), 148, lr.LR_PATH_TC)
            out.append(lr.LR_PATH_TC)
        except lr.LRError:
            pass
    return out


def lse_tol_for(lr, p, q, path):
    """The LSE bar: the stated one, or for int4 latents on tensor cores (fp16 operands)
    the rounding bound derived in helpers.fp16_operand_lse_bound."""
    if path == lr.LR_PATH_TC and p.quant_bits == 4:
        return H.decode_lse_bound(p, q)
    return None


def _sharp(p):
    f = H.sharp_factor(p)
    return p.store(H.stored_value(p, p.q) * f)


# ----------------------------------------------------------------------------
# per-workload parity (small variants)
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("kind", ["tiny", "qwen4k", "qwen16k", "hybrid"])
@pytest.mark.parametrize("sharp", [False, True])
def test_decode_parity(lib, kind, sharp):
    p = synth.small_variant(kind)
    c = H.fill_cache(lib, p)
    q = _sharp(p) if sharp else p.q
    ref, ref_lse = H.oracle_decode(p, q)
    for path in paths(lib, p):
        lib.lr_cache_set_path(c, path)
        got, lse = H.gpu_decode(lib, p, c, q)
        H.compare(p, got, ref, lse, ref_lse, tag=f"{kind} sharp={sharp} path={path}",
                  lse_tol=lse_tol_for(lib, p, q, path))


@pytest.mark.parametrize("layer", [0, 5, 4, 11, 12])
def test_decode_parity_prerope(lib, layer):
    """Keys stored before RoPE, rebuilt and rotated per tile (CUDA cores, and tensor cores
    for each KV-head pair).  Ranks of these layers: (256, 384), (128, 128), (400, 224),
    (448, 256), (192, 448) — partial last chunks, the largest ranks, r_k != r_v."""
    p = synth.small_variant("qwen32k", layer=layer, length=300)
    c = H.fill_cache(lib, p)
    for q in (p.q, _sharp(p)):
        ref, ref_lse = H.oracle_decode(p, q)
        for path in paths(lib, p):
            lib.lr_cache_set_path(c, path)
            got, lse = H.gpu_decode(lib, p, c, q)
            H.compare(p, got, ref, lse, ref_lse, tag=f"prerope layer={layer} path={path}",
                      lse_tol=lse_tol_for(lib, p, q, path))



def test_tiny_from_exact_keys_via_append(lib):
    """Config-1 path through lr_kv_append: the library projects K and V itself."""
    import torch
    p = synth.make_tiny()
    c = lib.lr_cache_create(H.desc_for(lib, p), H.to_dev(p, p.A_k), H.to_dev(p, p.B_k),
                            H.to_dev(p, p.A_v), H.to_dev(p, p.B_v))
    K, V = p.extra["K"], p.extra["V"]
    for t in range(K.shape[1]):
        lib.lr_kv_append(c, torch.from_numpy(K[:, t].copy()).cuda(), torch.from_numpy(V[:, t].copy()).cuda())
    zk = attention.project_latent(K, p.A_k)
    zv = attention.project_latent(V, p.A_v)
    ref, ref_lse = attention.decode(p.q.astype(np.float64), zk, zv, p.B_k, p.B_v, 1)
    got, lse = H.gpu_decode(lib, p, c)
    H.compare(p, got, ref, lse, ref_lse, tag="tiny append")


# ----------------------------------------------------------------------------
# bit-exact storage
# ----------------------------------------------------------------------------


def _read_int4(lib, p, c, n):
    v = lib.lr_cache_view_get(c)
    ck, pk = H.int4_token_major(lib, v, p.batch, "k")
    cv, pv = H.int4_token_major(lib, v, p.batch, "v")
    return ck[:, :n], pk[:, :n], cv[:, :n], pv[:, :n]


def _params_word(scale, zero):
    return scale.view(np.uint16).astype(np.uint32) | (zero.view(np.uint16).astype(np.uint32) << 16)


@pytest.mark.parametrize("layer", [None, 5, 4])
def test_int4_fill_bit_exact(lib, layer):
    if layer is None:
        p = synth.small_variant("qwen16k", length=333)
    else:
        p = synth.small_variant("qwen32k", layer=layer, length=333)
    c = H.fill_cache(lib, p, chunk=100)
    ck, pk, cv, pv = _read_int4(lib, p, c, p.hist_len)
    for z, codes, params in ((p.z_k, ck, pk), (p.z_v, cv, pv)):
        w, s, zz = quant.quantize_and_pack(z)
        assert np.array_equal(codes, w)
        assert np.array_equal(params, _params_word(s, zz))


def test_int4_quantiser_edge_cases_bit_exact(lib):
    """Hand-built groups: constant, ramp, ties, signed zeros, extreme spreads."""
    import torch
    r = 48
    rows = []
    rows.append(np.full(r, 3.25))
    rows.append(np.concatenate([np.arange(32), 100 + np.arange(16)]))
    x = np.zeros(r); x[0], x[1] = 0.0, 15.0; x[2:16] = np.arange(14) + 0.5; rows.append(x)
    x = np.zeros(r); x[::2] = -0.0; rows.append(x)
    rows.append(np.linspace(-7.5, 0.0, r))
    rows.append(np.concatenate([np.full(31, 1e-30), [2e-30], np.full(16, -5.0)]))
    rows.append(np.concatenate([[-60000.0, 60000.0], np.zeros(30), np.linspace(-1, 1, 16)]))
    rng = np.random.default_rng(0)
    rows.append(rng.standard_normal(r) * 1e3)
    z = np.stack(rows).astype(np.float32)[None]            # [1][n][r]
    n = z.shape[1]
    desc = lib.make_desc(1, 2, 1, 64, r, r, n + 4, quant_bits=4, dtype=lib.LR_F32)
    B = torch.zeros((r, 64), dtype=torch.float32, device="cuda")
    c = lib.lr_cache_create(desc, None, B, None, B)
    zt = torch.from_numpy(z).cuda()
    lib.lr_kv_append_latent(c, zt, zt)
    v = lib.lr_cache_view_get(c)
    codes, params = H.int4_token_major(lib, v, 1, "k")
    codes, params = codes[:, :n], params[:, :n]
    w, s, zz = quant.quantize_and_pack(z)
    assert np.array_equal(codes, w)
    assert np.array_equal(params, _params_word(s, zz))


def test_append_projection_and_quantiser_agree(lib):
    """lr_kv_append projects in fp32 on the GPU; an fp32-latent cache exposes the projected
    values, an int4 cache built from the same inputs must hold exactly the oracle's codes
    of those values, and the projection must match the fp64 oracle projection."""
    import torch
    rng = np.random.default_rng(3)
    Bsz, Hkv, d, r, n = 3, 2, 64, 80, 21
    D = Hkv * d
    A = rng.standard_normal((D, r)).astype(np.float32) / 8
    Bm = rng.standard_normal((r, D)).astype(np.float32)
    ks = rng.standard_normal((n, Bsz, D)).astype(np.float32)
    vs = rng.standard_normal((n, Bsz, D)).astype(np.float32)
    caches = {}
    for qb in (0, 4):
        desc = lib.make_desc(Bsz, 4, Hkv, d, r, r, n + 3, quant_bits=qb, dtype=lib.LR_F32)
        At, Bt = torch.from_numpy(A).cuda(), torch.from_numpy(Bm).cuda()
        c = lib.lr_cache_create(desc, At, Bt, At, Bt)
        for t in range(n):
            lib.lr_kv_append(c, torch.from_numpy(ks[t]).cuda(), torch.from_numpy(vs[t]).cuda())
        caches[qb] = c
    v = lib.lr_cache_view_get(caches[0])
    zk = lib.copy_view(v.z_k, (Bsz, v.capacity, r), "<f4").cpu().numpy()[:, :n]
    ref = attention.project_latent(ks.transpose(1, 0, 2), A)
    bound = 1e-6 * np.abs(ks).transpose(1, 0, 2) @ np.abs(A) + 1e-30
    assert np.all(np.abs(zk - ref) <= bound * 8)
    vq = lib.lr_cache_view_get(caches[4])
    codes, params = H.int4_token_major(lib, vq, Bsz, "k")
    codes, params = codes[:, :n], params[:, :n]
    w, s, zz = quant.quantize_and_pack(zk)
    assert np.array_equal(codes, w) and np.array_equal(params, _params_word(s, zz))
    assert lib.lr_cache_get_len(caches[4]) == (n, n, 0)


def test_window_ring_and_fold_indexing(lib):
    """Ring slot t % (W+1) holds token t exactly; folded tokens land in history slots in
    order; lengths follow the sliding fold."""
    import torch
    p = synth.small_variant("hybrid", hist_len=0, win_len=0, window=8, batch=2)
    c = lib.lr_cache_create(H.desc_for(lib, p, capacity=64), H.to_dev(p, p.A_k), H.to_dev(p, p.B_k),
                            H.to_dev(p, p.A_v), H.to_dev(p, p.B_v))
    D = p.kv_dim
    toks = []
    for t in range(20):
        k, v = synth.hybrid_token("hybrid", 0, t, 2, D, H.stored_value(p, p.B_k), H.stored_value(p, p.B_v))
        kb, vb = synth.bf16_bits(k), synth.bf16_bits(v)
        toks.append((kb, vb))
        lib.lr_kv_append(c, H.to_dev(p, kb), H.to_dev(p, vb))
        L, hl, wl = lib.lr_cache_get_len(c)
        assert (L, hl, wl) == (t + 1, max(0, t + 1 - 8), min(t + 1, 8))
    v = lib.lr_cache_view_get(c)
    ring = lib.copy_view(v.win_k, (2, v.window_slots, D), "<i2").cpu().numpy().view(np.uint16)
    for t in range(12, 20):
        assert np.array_equal(ring[:, t % 9], toks[t][0])
    zk = lib.copy_view(v.z_k, (2, v.capacity, p.rank_k), "<i2").cpu().numpy().view(np.uint16)[:, :12]
    # folded history slot t holds bf16(k_t A_k); compare within one bf16 ulp of the fp64 value
    A = H.stored_value(p, p.A_k)
    for t in range(12):
        z64 = attention.project_latent(H.stored_value(p, toks[t][0]), A)
        got = H.bf16_bits_to_f64(zk[:, t])
        ulp = np.abs(quant.round_to_bf16(z64)) * 2.0 ** -7 + 1e-30
        assert np.all(np.abs(got - z64) <= ulp)


def test_hybrid_steps_fold_and_sync(lib):
    """iS-KV stepping: appends that fold, decode after each, a basis sync with B' = R^T B,
    and the drift the sync prevents."""
    import torch
    p = synth.small_variant("hybrid", hist_len=300, batch=2)
    c = H.fill_cache(lib, p, capacity=p.length + 64)
    sim = iskv.WindowedCacheSim(H.stored_value(p, p.A_k), H.stored_value(p, p.B_k),
                                H.stored_value(p, p.A_v), H.stored_value(p, p.B_v),
                                p.n_kv_heads, p.window, "bf16")
    sim.fill_history(H.oracle_latents(p, p.z_k), H.oracle_latents(p, p.z_v))
    for t in range(p.win_len):
        sim.append(H.stored_value(p, p.win_k[:, t]), H.stored_value(p, p.win_v[:, t]))
    D = p.kv_dim
    q = _sharp(p)
    qv = H.stored_value(p, q)
    for step in range(3):
        k, v = synth.hybrid_token("hybrid", 0, 10_000 + step, p.batch, D,
                                  H.stored_value(p, p.B_k), H.stored_value(p, p.B_v), noise=1e-2)
        kb, vb = synth.bf16_bits(k), synth.bf16_bits(v)
        lib.lr_kv_append(c, H.to_dev(p, kb), H.to_dev(p, vb))
        sim.append(H.stored_value(p, kb), H.stored_value(p, vb))
        ref, ref_lse = sim.decode(qv)
        got, lse = H.gpu_decode(lib, p, c, q)
        H.compare(p, got, ref, lse, ref_lse, tag=f"hybrid step {step}")
    Rk = synth.sync_rotation(0, 0, p.rank_k, "k")
    Rv = synth.sync_rotation(0, 0, p.rank_v, "v")
    Bk_new = p.store(Rk.T @ H.stored_value(p, p.B_k))
    Bv_new = p.store(Rv.T @ H.stored_value(p, p.B_v))
    Ak_new = p.store(H.stored_value(p, p.A_k) @ Rk)
    Av_new = p.store(H.stored_value(p, p.A_v) @ Rv)
    before, _ = H.gpu_decode(lib, p, c, q)
    lib.lr_basis_sync(c, torch.from_numpy(Rk.astype(np.float32)).cuda(),
                      torch.from_numpy(Rv.astype(np.float32)).cuda(), H.to_dev(p, Bk_new),
                      H.to_dev(p, Bv_new), H.to_dev(p, Ak_new), H.to_dev(p, Av_new))
    sim.sync(Rk.astype(np.float32), Rv.astype(np.float32), H.stored_value(p, Bk_new),
             H.stored_value(p, Bv_new), H.stored_value(p, Ak_new), H.stored_value(p, Av_new))
    ref, ref_lse = sim.decode(qv)
    got, lse = H.gpu_decode(lib, p, c, q)
    H.compare(p, got, ref, lse, ref_lse, tag="after sync")
    # invariance: the output after the sync stays close to the one before
    assert np.max(np.abs(got - before)) <= 0.05 * np.max(np.abs(before))
    # keep stepping after the sync (folds use the new A)
    for step in range(3, 5):
        k, v = synth.hybrid_token("hybrid", 0, 10_000 + step, p.batch, D,
                                  H.stored_value(p, Bk_new), H.stored_value(p, Bv_new), noise=1e-2)
        kb, vb = synth.bf16_bits(k), synth.bf16_bits(v)
        lib.lr_kv_append(c, H.to_dev(p, kb), H.to_dev(p, vb))
        sim.append(H.stored_value(p, kb), H.stored_value(p, vb))
        ref, ref_lse = sim.decode(qv)
        got, lse = H.gpu_decode(lib, p, c, q)
        H.compare(p, got, ref, lse, ref_lse, tag=f"hybrid step {step} after sync")


def test_sync_drift_without_rotation(lib):
    """Installing B' = R^T B without rotating the stored coordinates moves the output
    (the drift iS-KV describes); rotating them restores it."""
    import torch
    p = synth.small_variant("hybrid", hist_len=400, batch=1)
    q = _sharp(p)
    c0 = H.fill_cache(lib, p)
    base, _ = H.gpu_decode(lib, p, c0, q)
    Rk = synth.sync_rotation(0, 1, p.rank_k, "k")
    Bk_new = p.store(Rk.T @ H.stored_value(p, p.B_k))
    c1 = H.fill_cache(lib, p)
    lib.lr_basis_sync(c1, None, None, H.to_dev(p, Bk_new), None, None, None)
    drift, _ = H.gpu_decode(lib, p, c1, q)
    c2 = H.fill_cache(lib, p)
    lib.lr_basis_sync(c2, torch.from_numpy(Rk.astype(np.float32)).cuda(), None, H.to_dev(p, Bk_new),
                      None, None, None)
    synced, _ = H.gpu_decode(lib, p, c2, q)
    scale = np.max(np.abs(base))
    assert np.max(np.abs(drift - base)) > 0.1 * scale
    assert np.max(np.abs(synced - base)) < 0.03 * scale


def test_sync_identity_is_bit_exact(lib):
    import torch
    p = synth.small_variant("hybrid", hist_len=200, batch=1)
    c = H.fill_cache(lib, p)
    v = lib.lr_cache_view_get(c)
    before = lib.copy_view(v.z_k, (1, v.capacity, p.rank_k), "<i2").cpu().numpy()
    I = torch.eye(p.rank_k, dtype=torch.float32, device="cuda")
    lib.lr_basis_sync(c, I, I, None, None, None, None)
    after = lib.copy_view(v.z_k, (1, v.capacity, p.rank_k), "<i2").cpu().numpy()
    assert np.array_equal(before, after)


@pytest.mark.parametrize("which,hist,batch", [("kv", 700, 2), ("k", 700, 2), ("v", 700, 2),
                                              ("kv", 5000, 4), ("v", 5000, 4)])
def test_sync_tensor_core_matches_oracle_and_cuda_cores(lib, which, hist, batch):
    """The tensor-core sync (bf16 latents, r <= 256) against the oracle's rounded fp64
    Z R and against the CUDA-core sync: several 128-token tiles plus a ragged tail,
    several sequences, one side or both; at 5000 tokens x 4 sequences there are more
    tiles than SMs, so each CTA runs several tiles through its two tile buffers and two
    accumulators."""
    import torch
    p = synth.small_variant("hybrid", hist_len=hist, batch=batch)
    c_tc, c_simt = H.fill_cache(lib, p), H.fill_cache(lib, p)
    lib.lr_cache_set_path(c_simt, lib.LR_PATH_SIMT)
    Rk = synth.sync_rotation(0, 3, p.rank_k, "k").astype(np.float32)
    Rv = synth.sync_rotation(0, 3, p.rank_v, "v").astype(np.float32)
    rk = torch.from_numpy(Rk).cuda() if "k" in which else None
    rv = torch.from_numpy(Rv).cuda() if "v" in which else None
    for c in (c_tc, c_simt):
        lib.lr_basis_sync(c, rk, rv, None, None, None, None)
    torch.cuda.synchronize()
    n = p.hist_len
    for side, R, on in (("k", Rk, "k" in which), ("v", Rv, "v" in which)):
        z0 = H.oracle_latents(p, p.z_k if side == "k" else p.z_v)        # stored bf16 values
        ref = synth.bf16_bits(z0 @ R.astype(np.float64)) if on else synth.bf16_bits(z0)
        got = []
        for c in (c_tc, c_simt):
            v = lib.lr_cache_view_get(c)
            z = lib.copy_view(v.z_k if side == "k" else v.z_v, (p.batch, v.capacity, p.rank_k), "<i2")
            got.append(z.cpu().numpy().view(np.uint16)[:, :n])
        rv64 = synth.bf16_to_f64(ref)
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(rv64), 1e-30))) - 7)   # bf16 spacing at ref
        # rounding bound of the computed product before its bf16 store: R split into bf16
        # hi + lo leaves <= 2^-18 |R| per entry, and fp32 accumulation of 2r terms adds
        # <= 2r 2^-24 sum|z R|; 2^-14 sum_k |z_k| |R_kn| covers both (cancellations near zero
        # make ulps of the result meaningless there)
        mag = (np.abs(z0) @ np.abs(R.astype(np.float64))) if on else np.zeros_like(rv64)
        bound = ulp + 2.0 ** -14 * mag
        for name, g in zip(("tensor cores", "cuda cores"), got):
            err = np.abs(synth.bf16_to_f64(g) - rv64)
            assert np.all(err <= bound), f"{side} {name}: {np.max(err / bound):.2f} x bound"
            assert np.mean(err > 0) < 0.01, f"{side} {name}: {np.mean(err > 0):.4f} of elements differ"
    assert lib.lr_device_error(c_tc) == 0


# ----------------------------------------------------------------------------
@pytest.mark.parametrize("layer", [0, 5, 4])
def test_decode_parity_int4_postrope(lib, layer):
    """The 28-layer int4 cache with keys stored after RoPE (q~ path, tensor cores where
    supported): per-layer ranks (256, 384), (128, 128), (400, 224) — partial int4 groups,
    r_k != r_v, several 128-rank chunks."""
    p = synth.small_variant("qwen32k", layer=layer, length=700, rope=False)
    c = H.fill_cache(lib, p)
    for q in (p.q, _sharp(p)):
        ref, ref_lse = H.oracle_decode(p, q)
        for path in paths(lib, p):
            lib.lr_cache_set_path(c, path)
            got, lse = H.gpu_decode(lib, p, c, q)
            H.compare(p, got, ref, lse, ref_lse, tag=f"int4 post-RoPE layer={layer} path={path}",
                      lse_tol=lse_tol_for(lib, p, q, path))


# invariants and edge cases
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("kind", ["qwen4k", "qwen16k", "qwen32k"])
def test_split_count_invariance(lib, kind):
    p = synth.small_variant(kind, length=1000)
    c = H.fill_cache(lib, p)
    q = _sharp(p)
    for path in paths(lib, p):
        outs = []
        for s in ((1, 2, 7, 60) if path == lib.LR_PATH_SIMT else (1, 2, 3, 8)):
            lib.lr_cache_set_path(c, path, s)
            got, lse = H.gpu_decode(lib, p, c, q)
            outs.append((got, lse))
        ref = outs[0]
        # fp16 probabilities (int4 on tensor cores) are rounded relative to each split's
        # own running max, so l moves by up to 2^-11 relative per side
        ltol = 2.0 ** -10 if (path == lib.LR_PATH_TC and p.quant_bits == 4) else 1e-4
        for got, lse in outs[1:]:
            assert np.max(np.abs(got - ref[0])) <= 2e-2 * np.max(np.abs(ref[0])) + 1e-6
            assert np.max(np.abs(lse - ref[1])) <= ltol


@pytest.mark.parametrize("length", [1, 127, 128, 129, 255, 257])
def test_tile_edges(lib, length):
    """Lengths around the 128-token tile: T=1 returns v^ (up to rounding), ragged tails."""
    p = synth.small_variant("qwen4k", length=length, batch=2)
    c = H.fill_cache(lib, p)
    q = _sharp(p)
    ref, ref_lse = H.oracle_decode(p, q)
    for path in paths(lib, p):
        lib.lr_cache_set_path(c, path)
        got, lse = H.gpu_decode(lib, p, c, q)
        H.compare(p, got, ref, lse, ref_lse, tag=f"T={length} path={path}")


@pytest.mark.parametrize("length", [1, 127, 128, 129, 255, 257, 384])
def test_tile_edges_int4(lib, length):
    """int4 latents around the 128-token tile (partial bulk copies of codes and of the
    unaligned {scale, zero} spans; zero-filled tail rows)."""
    p = synth.small_variant("qwen16k", length=length, batch=3)
    c = H.fill_cache(lib, p)
    q = _sharp(p)
    ref, ref_lse = H.oracle_decode(p, q)
    for path in paths(lib, p):
        lib.lr_cache_set_path(c, path)
        got, lse = H.gpu_decode(lib, p, c, q)
        H.compare(p, got, ref, lse, ref_lse, tag=f"int4 T={length} path={path}",
                  lse_tol=lse_tol_for(lib, p, q, path))


@pytest.mark.parametrize("length", [1, 127, 128, 129, 257])
def test_tile_edges_int4_prerope(lib, length):
    """Keys before RoPE around the 128-token tile: the rotation positions of ragged tiles
    and of later splits, zero-filled tail rows."""
    p = synth.small_variant("qwen32k", layer=0, length=length, batch=3)
    c = H.fill_cache(lib, p)
    q = _sharp(p)
    ref, ref_lse = H.oracle_decode(p, q)
    for path in paths(lib, p):
        lib.lr_cache_set_path(c, path)
        got, lse = H.gpu_decode(lib, p, c, q)
        H.compare(p, got, ref, lse, ref_lse, tag=f"int4 pre-RoPE T={length} path={path}",
                  lse_tol=lse_tol_for(lib, p, q, path))


def test_gqa_identical_queries_identical_outputs(lib):
    p = synth.small_variant("qwen4k", length=500)
    q = p.q.copy()
    q[:, 1:7] = q[:, 0:1]                  # heads 0..6 share KV head 0
    c = H.fill_cache(lib, p)
    for path in paths(lib, p):
        lib.lr_cache_set_path(c, path)
        got, _ = H.gpu_decode(lib, p, c, q)
        for j in range(1, 7):
            assert np.array_equal(got[:, j], got[:, 0])


def test_window_only_and_history_only(lib):
    p = synth.small_variant("hybrid", hist_len=0, win_len=50)
    c = H.fill_cache(lib, p)
    ref, ref_lse = H.oracle_decode(p)
    got, lse = H.gpu_decode(lib, p, c)
    H.compare(p, got, ref, lse, ref_lse, tag="window only")
    p2 = synth.small_variant("hybrid", hist_len=200, win_len=0)
    c2 = H.fill_cache(lib, p2)
    ref, ref_lse = H.oracle_decode(p2)
    got, lse = H.gpu_decode(lib, p2, c2)
    H.compare(p2, got, ref, lse, ref_lse, tag="history only")


@pytest.mark.parametrize("head_dim,rank", [(24, 32), (40, 64), (256, 64), (64, 64)])
def test_window_head_dims(lib, head_dim, rank):
    """The exact window at head dims whose 16-byte row vectors do or do not divide the
    window kernel's block (its two copy walks), with columns past 128 (d = 256) and a ring
    that wraps (the window starts at slot hist_len mod (W + 1))."""
    p = synth.make_hybrid(batch=2, hist_len=150, window=100, rank=rank, n_q_heads=4, n_kv_heads=2,
                          head_dim=head_dim)
    p = dataclasses.replace(p, q=p.store(H.stored_value(p, p.q) * H.sharp_factor(p)))
    c = H.fill_cache(lib, p)
    ref, ref_lse = H.oracle_decode(p)
    got, lse = H.gpu_decode(lib, p, c)
    H.compare(p, got, ref, lse, ref_lse, tag=f"window d={head_dim}")
    lib.lr_cache_destroy(c)


def test_capacity_and_argument_errors(lib):
    import torch
    p = synth.small_variant("qwen4k", length=10, batch=1)
    c = H.fill_cache(lib, p, capacity=11)
    k = torch.zeros((1, p.kv_dim), dtype=torch.bfloat16, device="cuda")
    lib.lr_kv_append(c, k, k)
    with pytest.raises(lib.LRError) as e:
        lib.lr_kv_append(c, k, k)
    assert e.value.status == lib.LR_ERR_CAPACITY
    z = torch.zeros((1, 1, p.rank_k), dtype=torch.float32, device="cuda")
    with pytest.raises(lib.LRError) as e:
        lib.lr_kv_append_latent(c, z, z)
    assert e.value.status == lib.LR_ERR_CAPACITY
    empty = lib.lr_cache_create(H.desc_for(lib, p), H.to_dev(p, p.A_k), H.to_dev(p, p.B_k),
                                H.to_dev(p, p.A_v), H.to_dev(p, p.B_v))
    q = H.to_dev(p, p.q)
    with pytest.raises(lib.LRError) as e:
        lib.lr_attn_decode(empty, q, torch.empty_like(q))
    assert e.value.status == lib.LR_ERR_INVALID_ARG
    assert lib.lr_device_error(c) == 0


def test_truncate_replays_same_step(lib):
    p = synth.small_variant("qwen4k", length=600)
    c = H.fill_cache(lib, p)
    first, _ = H.gpu_decode(lib, p, c)
    k = H.to_dev(p, synth.bf16_bits(np.ones((p.batch, p.kv_dim))))
    for _ in range(3):
        lib.lr_kv_append(c, k, k)
        lib.lr_cache_truncate(c, p.length)
    again, _ = H.gpu_decode(lib, p, c)
    assert np.array_equal(first, again)


@pytest.mark.parametrize("win_len", [50, 128])
def test_truncate_undoes_last_append_with_window(lib, win_len):
    """A windowed cache can drop the token of its last append (the ring's spare slot keeps
    the folded token): window not yet full (no fold) and full (fold)."""
    p = synth.small_variant("hybrid", hist_len=300, win_len=win_len)
    c = H.fill_cache(lib, p)
    first, first_lse = H.gpu_decode(lib, p, c)
    n0 = lib.lr_cache_get_len(c)
    k, v = synth.hybrid_token("undo", 0, 0, p.batch, p.kv_dim, H.stored_value(p, p.B_k), H.stored_value(p, p.B_v))
    for _ in range(2):
        lib.lr_kv_append(c, H.to_dev(p, p.store(k)), H.to_dev(p, p.store(v)))
        assert lib.lr_cache_get_len(c) != n0
        lib.lr_cache_truncate(c, n0[0])
        assert lib.lr_cache_get_len(c) == n0
        again, again_lse = H.gpu_decode(lib, p, c)
        assert np.array_equal(first, again) and np.array_equal(first_lse, again_lse)
    with pytest.raises(lib.LRError) as e:
        lib.lr_cache_truncate(c, n0[0] - 1)           # nothing left to undo
    assert e.value.status == lib.LR_ERR_UNSUPPORTED


@pytest.mark.parametrize("kind", ["tiny", "qwen4k", "qwen16k", "hybrid"])
def test_decode_step_equals_append_then_decode(lib, kind):
    """lr_decode_step is lr_kv_append followed by lr_attn_decode, bit for bit."""
    import torch
    p = synth.small_variant(kind)
    c1, c2 = H.fill_cache(lib, p), H.fill_cache(lib, p)
    D = p.kv_dim
    q = _sharp(p)
    for step in range(3):
        k, v = synth.hybrid_token("step", 0, step, p.batch, D, H.stored_value(p, p.B_k), H.stored_value(p, p.B_v))
        kd, vd, qd = H.to_dev(p, p.store(k)), H.to_dev(p, p.store(v)), H.to_dev(p, q)
        o1, o2 = torch.empty_like(qd), torch.empty_like(qd)
        l1 = torch.empty((p.batch, p.n_q_heads), dtype=torch.float32, device="cuda")
        l2 = torch.empty_like(l1)
        lib.lr_kv_append(c1, kd, vd)
        lib.lr_attn_decode(c1, qd, o1, l1)
        lib.lr_decode_step(c2, kd, vd, qd, o2, l2)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        assert lib.lr_cache_get_len(c1) == lib.lr_cache_get_len(c2)


def test_decode_step_window_paths_equal_append_then_decode(lib):
    """The fused step computes the exact window ahead of its own kernels, from the ring rows of
    earlier steps and the step's own k, v and q; right after a standalone append of the same
    cache it waits before reading the ring.  Both, with a window of two 128-token rounds that
    fills up and then folds, equal lr_kv_append + lr_attn_decode bit for bit, step by step."""
    import torch
    p = synth.small_variant("hybrid", hist_len=300, window=200, win_len=190, batch=2)
    c1, c2 = H.fill_cache(lib, p, capacity=600), H.fill_cache(lib, p, capacity=600)
    D = p.kv_dim
    q = _sharp(p)
    qd = H.to_dev(p, q)
    # per step: True = lr_decode_step on c2, False = lr_kv_append + lr_attn_decode on c2 too
    plan = [True, True, False, True, False, False, True] + [True] * 7
    for step, fused in enumerate(plan):
        k, v = synth.hybrid_token("wstep", 0, step, p.batch, D, H.stored_value(p, p.B_k), H.stored_value(p, p.B_v))
        kd, vd = H.to_dev(p, p.store(k)), H.to_dev(p, p.store(v))
        o1, o2 = torch.empty_like(qd), torch.empty_like(qd)
        l1 = torch.empty((p.batch, p.n_q_heads), dtype=torch.float32, device="cuda")
        l2 = torch.empty_like(l1)
        lib.lr_kv_append(c1, kd, vd)
        lib.lr_attn_decode(c1, qd, o1, l1)
        if fused:
            lib.lr_decode_step(c2, kd, vd, qd, o2, l2)
        else:
            lib.lr_kv_append(c2, kd, vd)
            lib.lr_attn_decode(c2, qd, o2, l2)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2), f"step {step}"
        assert lib.lr_cache_get_len(c1) == lib.lr_cache_get_len(c2)
    assert lib.lr_cache_get_len(c1)[2] == 200          # the window filled and folded
    lib.lr_cache_destroy(c1)
    lib.lr_cache_destroy(c2)


@pytest.mark.parametrize("hq,hkv", [(8, 2), (12, 3), (16, 1), (28, 4)])
def test_decode_parity_prerope_head_shapes(lib, hq, hkv):
    """Keys before RoPE on tensor cores for other group sizes and KV-head counts: pairs of KV
    heads (Hkv even) or single heads (Hkv odd), up to 16 query heads per KV head (the
    score MMA's N); against the oracle, with the CUDA-core path alongside."""
    D = hkv * 128
    p = synth.make_qwen("qwen32k", seed=3, batch=2, length=300, rank=min(192, D), quant_bits=4, rope=True,
                        n_q_heads=hq, n_kv_heads=hkv, rank_v=min(160, D - 16))
    c = H.fill_cache(lib, p)
    assert lib.LR_PATH_TC in paths(lib, p)
    for q in (p.q, _sharp(p)):
        ref, ref_lse = H.oracle_decode(p, q)
        for path in paths(lib, p):
            lib.lr_cache_set_path(c, path)
            got, lse = H.gpu_decode(lib, p, c, q)
            H.compare(p, got, ref, lse, ref_lse, tag=f"prerope Hq={hq} Hkv={hkv} path={path}",
                      lse_tol=lse_tol_for(lib, p, q, path))
    lib.lr_cache_destroy(c)
