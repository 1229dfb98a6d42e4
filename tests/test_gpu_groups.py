"""Latent groups: a cache whose KV heads are split into g groups, each with its own latents and
bases (g = n_kv_heads: one latent per KV head, the grouped layout of Palu that the ai4snews
digest's Interpretation section compares against).  The oracle reconstructs every key and
value through the block-diagonal basis that the per-group bases form, so it checks the
grouping, the fill, the projection of appended tokens and the per-group basis sync."""
import dataclasses

import numpy as np
import pytest

import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _blockdiag(blocks):
    g = len(blocks)
    r, c = blocks[0].shape
    out = np.zeros((g * r, g * c))
    for i, b in enumerate(blocks):
        out[i * r:(i + 1) * r, i * c:(i + 1) * c] = b
    return out


def grouped_problem(g, r, quant_bits, batch=2, length=500, n_q_heads=28, n_kv_heads=4, seed=0):
    """Per-group Haar bases (rows / sqrt(r), A = r B^T) and latents N(0,1) i^-0.7 per group."""
    rng = synth.rng_for("groups", f"g{g}r{r}q{quant_bits}", seed)
    D, d = n_kv_heads * 128, 128
    Dg = D // g
    Bk = [synth.haar_orthonormal(rng, r, Dg) / np.sqrt(r) for _ in range(g)]
    Bv = [synth.haar_orthonormal(rng, r, Dg) / np.sqrt(r) for _ in range(g)]
    sig = synth.spectrum(r, 0.7)
    zk = np.concatenate([rng.standard_normal((batch, length, r)) * sig for _ in range(g)], axis=2)
    zv = np.concatenate([rng.standard_normal((batch, length, r)) * sig for _ in range(g)], axis=2)
    q = rng.standard_normal((batch, n_q_heads, d)) / np.sqrt(128.0)
    bf = synth.bf16_bits
    p = synth.Problem("groups", batch, n_q_heads, n_kv_heads, d, g * r, g * r, "bf16", quant_bits, False, 1e6,
                      0, length, bf(_blockdiag([r * b.T for b in Bk])), bf(_blockdiag(Bk)),
                      bf(_blockdiag([r * b.T for b in Bv])), bf(_blockdiag(Bv)),
                      zk.astype(np.float32), zv.astype(np.float32), bf(q))
    compact = dict(A_k=bf(np.stack([r * b.T for b in Bk])), B_k=bf(np.stack(Bk)),
                   A_v=bf(np.stack([r * b.T for b in Bv])), B_v=bf(np.stack(Bv)))
    return p, compact


def fill(lib, p, compact, g, r):
    import torch
    desc = lib.make_desc(p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, r, r, p.length + 8,
                         quant_bits=p.quant_bits, latent_groups=g)
    c = lib.lr_cache_create(desc, *(H.to_dev(p, compact[k]) for k in ("A_k", "B_k", "A_v", "B_v")))
    lib.lr_kv_append_latent(c, torch.from_numpy(np.ascontiguousarray(p.z_k)).cuda(),
                            torch.from_numpy(np.ascontiguousarray(p.z_v)).cuda())
    return c


@pytest.mark.parametrize("g,r", [(4, 64), (2, 96), (4, 112)])
@pytest.mark.parametrize("quant_bits", [0, 4])
def test_grouped_decode_matches_oracle(lib, g, r, quant_bits):
    p, compact = grouped_problem(g, r, quant_bits)
    c = fill(lib, p, compact, g, r)
    view = lib.lr_cache_view_get(c)
    B_full = lib.copy_view(view.B_k, (g * r, p.kv_dim), "<i2").cpu().numpy().view(np.uint16)
    assert np.array_equal(B_full, p.B_k)                       # the block-diagonal basis, zeros included
    for q in (p.q, p.store(H.stored_value(p, p.q) * H.sharp_factor(p))):
        ref, ref_lse = H.oracle_decode(p, q)
        for path in (lib.LR_PATH_SIMT, lib.LR_PATH_AUTO):
            lib.lr_cache_set_path(c, path)
            got, lse = H.gpu_decode(lib, p, c, q)
            tc = lib.lr_cache_plan(c).path == lib.LR_PATH_TC
            H.compare(p, got, ref, lse, ref_lse, tag=f"groups g={g} r={r} q{quant_bits} path={path}",
                      lse_tol=H.decode_lse_bound(p, q) if (tc and quant_bits == 4) else None)
    lib.lr_cache_destroy(c)


def test_grouped_append_projects_each_group_with_its_own_basis(lib):
    """lr_kv_append of exact tokens: each group's latent is its KV heads' keys times its own
    A block; the oracle projects with the block-diagonal A."""
    import torch
    g, r = 4, 64
    p, compact = grouped_problem(g, r, 0, length=200)
    c = fill(lib, p, compact, g, r)
    rng = np.random.default_rng(8)
    kx = rng.standard_normal((p.batch, p.kv_dim)) * 0.01
    vx = rng.standard_normal((p.batch, p.kv_dim)) * 0.01
    lib.lr_kv_append(c, H.to_dev(p, p.store(kx)), H.to_dev(p, p.store(vx)))
    torch.cuda.synchronize()
    view = lib.lr_cache_view_get(c)
    zk = lib.copy_view(view.z_k, (p.batch, p.length + 8, g * r), "<i2").cpu().numpy().view(np.uint16)
    from oracle import attention, quant
    want = quant.round_to_bf16(attention.project_latent(p.to_f64(p.store(kx)), p.to_f64(p.A_k)))
    got = synth.bf16_to_f64(zk[:, p.length])
    # fp32 accumulation in a different order than fp64: at most one bf16 step apart
    assert np.all(np.abs(got - want) <= 2.0 ** -7 * np.abs(want) + 1e-30)
    lib.lr_cache_destroy(c)


def test_grouped_sync_with_per_group_rotations_keeps_outputs(lib):
    """Per-group orthogonal R_i with B_i' = R_i^T B_i leave every reconstructed key and value
    unchanged: the decode after the sync matches the oracle of the unsynchronised cache."""
    import torch
    g, r = 4, 64
    p, compact = grouped_problem(g, r, 0, length=300)
    c = fill(lib, p, compact, g, r)
    ref, ref_lse = H.oracle_decode(p)
    rng = np.random.default_rng(4)
    R = np.stack([synth.haar_orthogonal(rng, r) for _ in range(g)])
    Bk = p.to_f64(compact["B_k"])
    Bv = p.to_f64(compact["B_v"])
    Bk_new = np.stack([R[i].T @ Bk[i] for i in range(g)])
    Bv_new = np.stack([R[i].T @ Bv[i] for i in range(g)])
    Rd = torch.from_numpy(R.astype(np.float32)).cuda()
    lib.lr_basis_sync(c, Rd, Rd, H.to_dev(p, p.store(Bk_new)), H.to_dev(p, p.store(Bv_new)))
    got, lse = H.gpu_decode(lib, p, c)
    # bf16 rounding of the rotated latents and of the new bases: the stated bars still hold
    H.compare(p, got, ref, lse, ref_lse, tag="groups after sync")
    lib.lr_cache_destroy(c)


@pytest.mark.parametrize("quant_bits", [0, 4])
def test_grouped_paged_equals_contiguous(lib, quant_bits):
    """Latent groups in a paged cache (shuffled block table): bit-identical to the contiguous
    grouped cache."""
    import torch
    g, r = 4, 64
    p, compact = grouped_problem(g, r, quant_bits, batch=3, length=600)
    cap = 640
    caches = []
    for paged in (False, True):
        desc = lib.make_desc(p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, r, r, cap,
                             quant_bits=quant_bits, latent_groups=g, page_tokens=128 if paged else 0,
                             n_pages=p.batch * (cap // 128) + 2 if paged else 0)
        c = lib.lr_cache_create(desc, *(H.to_dev(p, compact[k]) for k in ("A_k", "B_k", "A_v", "B_v")))
        if paged:
            perm = np.random.default_rng(4).permutation(p.batch * (cap // 128) + 2)[:p.batch * (cap // 128)]
            lib.lr_cache_set_block_table(c, perm.astype(np.int32).reshape(p.batch, cap // 128))
        lib.lr_kv_append_latent(c, torch.from_numpy(np.ascontiguousarray(p.z_k)).cuda(),
                                torch.from_numpy(np.ascontiguousarray(p.z_v)).cuda())
        caches.append(c)
    q = p.store(H.stored_value(p, p.q) * H.sharp_factor(p))
    (a, la), (b, lb) = (H.gpu_decode(lib, p, c, q) for c in caches)
    assert np.array_equal(a, b) and np.array_equal(la, lb)
    for c in caches:
        lib.lr_cache_destroy(c)
