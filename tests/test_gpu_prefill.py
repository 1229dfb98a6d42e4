"""Bulk prefill (lr_kv_prefill): the latents of a whole prompt from its exact keys and values,
on the tensor cores for bf16 caches.  Checked against the oracle's fp64 projection: bf16
latents within one bf16 step of the oracle's rounding (the fp32 sums run in another order),
int4 codes equal to the oracle's except where the fp32 value sits at a rounding boundary,
and the decode after the prefill within the parity bars; prefills that start inside an
8-token word of the rank-major value layout, ragged tiles and ranks above 256 included."""
import dataclasses

import numpy as np
import pytest

import synth
from oracle import attention, quant
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _tokens(p, n, seed):
    """Exact keys / values whose projections have the law of the stored latents: x = (g sigma) B
    plus 1% off-subspace noise."""
    rng = np.random.default_rng(seed)
    Bk, Bv = p.to_f64(p.B_k), p.to_f64(p.B_v)
    sk = synth.spectrum(p.rank_k, 0.7)
    sv = synth.spectrum(p.rank_v, 0.7)
    k = (rng.standard_normal((p.batch, n, p.rank_k)) * sk) @ Bk
    v = (rng.standard_normal((p.batch, n, p.rank_v)) * sv) @ Bv
    k = k + 1e-2 * np.abs(k).mean() * rng.standard_normal(k.shape)
    v = v + 1e-2 * np.abs(v).mean() * rng.standard_normal(v.shape)
    return p.store(k), p.store(v)


@pytest.mark.parametrize("quant_bits,rank", [(0, 256), (4, 352), (0, 448), (4, 128), (0, 48), (4, 48)])
@pytest.mark.parametrize("cuts", [[300], [13, 300], [64, 200]])
def test_prefill_matches_oracle_projection(lib, quant_bits, rank, cuts):
    import torch
    p0 = synth.make_qwen("qwen16k", batch=2, length=0, rank=rank, quant_bits=quant_bits)
    n = sum(cuts)
    kx, vx = _tokens(p0, n, seed=rank + n)
    desc = lib.make_desc(p0.batch, p0.n_q_heads, p0.n_kv_heads, p0.head_dim, rank, rank, n + 8,
                         quant_bits=quant_bits)
    c = lib.lr_cache_create(desc, H.to_dev(p0, p0.A_k), H.to_dev(p0, p0.B_k), H.to_dev(p0, p0.A_v),
                            H.to_dev(p0, p0.B_v))
    s = 0
    for m in cuts:                                  # several prefills; later ones start mid-word
        lib.lr_kv_prefill(c, H.to_dev(p0, np.ascontiguousarray(kx[:, s:s + m])),
                          H.to_dev(p0, np.ascontiguousarray(vx[:, s:s + m])))
        s += m
    torch.cuda.synchronize()
    assert lib.lr_cache_get_len(c) == (n, n, 0)
    # the oracle's projection of the same tokens
    zk = attention.project_latent(p0.to_f64(kx), p0.to_f64(p0.A_k))
    zv = attention.project_latent(p0.to_f64(vx), p0.to_f64(p0.A_v))
    view = lib.lr_cache_view_get(c)
    if quant_bits == 0:
        for ptr, z, x, A in ((view.z_k, zk, kx, p0.A_k), (view.z_v, zv, vx, p0.A_v)):
            got = synth.bf16_to_f64(lib.copy_view(ptr, (p0.batch, n + 8, rank), "<i2").cpu().numpy().view(np.uint16)[:, :n])
            want = quant.round_to_bf16(z)
            # one bf16 step, plus the fp32 summation error of a D-term dot product in any order
            # (which can move the value across a rounding boundary)
            fp32 = p0.kv_dim * 2.0 ** -24 * (np.abs(p0.to_f64(x)) @ np.abs(p0.to_f64(A)))
            assert np.all(np.abs(got - want) <= 2.0 ** -7 * np.abs(want) + 2 * fp32)
    else:
        for side, z in (("k", zk), ("v", zv)):
            codes, params = H.int4_token_major(lib, view, p0.batch, side)
            w, sc, zr = quant.quantize_and_pack(z.astype(np.float32))
            got = quant.unpack_nibbles(codes[:, :n])[..., :rank].astype(int)
            ref = quant.unpack_nibbles(w)[..., :rank].astype(int)
            diff = np.abs(got - ref)
            assert diff.max() <= 1, (side, diff.max())
            assert diff.mean() < 1e-3, (side, diff.mean())
    # decode over the prefilled cache, against the oracle of the oracle-projected latents
    p = dataclasses.replace(p0, hist_len=n, z_k=zk.astype(np.float32), z_v=zv.astype(np.float32))
    for q in (p.q, p.store(H.stored_value(p, p.q) * H.sharp_factor(p))):
        ref, ref_lse = H.oracle_decode(p, q)
        got, lse = H.gpu_decode(lib, p, c, q)
        H.compare(p, got, ref, lse, ref_lse, tag=f"prefill q{quant_bits} r={rank} cuts={cuts}",
                  lse_tol=H.decode_lse_bound(p, q) if quant_bits == 4 else None)
    lib.lr_cache_destroy(c)


def test_prefill_equals_appends_on_cuda_cores_for_fp32(lib):
    """fp32 caches take the per-token path: bit-identical to lr_kv_append one token at a time."""
    import torch
    p = synth.make_tiny()
    n = 40
    rng = np.random.default_rng(2)
    kx = rng.standard_normal((p.batch, n, p.kv_dim)).astype(np.float32)
    vx = rng.standard_normal((p.batch, n, p.kv_dim)).astype(np.float32)
    caches = []
    for bulk in (True, False):
        c = lib.lr_cache_create(H.desc_for(lib, p, capacity=n + 4), H.to_dev(p, p.A_k), H.to_dev(p, p.B_k),
                                H.to_dev(p, p.A_v), H.to_dev(p, p.B_v))
        if bulk:
            lib.lr_kv_prefill(c, torch.from_numpy(kx).cuda(), torch.from_numpy(vx).cuda())
        else:
            for t in range(n):
                lib.lr_kv_append(c, torch.from_numpy(np.ascontiguousarray(kx[:, t])).cuda(),
                                 torch.from_numpy(np.ascontiguousarray(vx[:, t])).cuda())
        caches.append(c)
    torch.cuda.synchronize()
    a, b = (lib.copy_view(lib.lr_cache_view_get(c).z_k, (p.batch, n + 4, p.rank_k), "<f4").cpu().numpy() for c in caches)
    assert np.array_equal(a, b)
    for c in caches:
        lib.lr_cache_destroy(c)


def test_prefill_refuses_windows_and_overflow(lib):
    import torch
    p = synth.small_variant("hybrid", batch=2, hist_len=10)
    c = H.fill_cache(lib, p)
    k = torch.zeros((p.batch, 4, p.kv_dim), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.LRError) as e:
        lib.lr_kv_prefill(c, k, k)
    assert e.value.status == lib.LR_ERR_UNSUPPORTED
    lib.lr_cache_destroy(c)
    p = synth.small_variant("qwen4k", batch=2, length=10)
    c = H.fill_cache(lib, p, capacity=12)
    k = torch.zeros((p.batch, 4, p.kv_dim), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.LRError) as e:
        lib.lr_kv_prefill(c, k, k)
    assert e.value.status == lib.LR_ERR_CAPACITY
    lib.lr_cache_destroy(c)
