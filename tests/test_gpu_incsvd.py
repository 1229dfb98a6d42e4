"""GPU block-incremental SVD update (lr_basis_update) against the oracle's block update.

The oracle (oracle/incsvd.py, pinned on the CPU by Eckart-Young on the stacked matrix) and the
GPU take the same fp32 inputs; both compute in fp64, the GPU returns fp32 / dtype results.
Compared: the new Gram diagonal (eigenvalues), the new basis rows and the sync rotation up to
the sign of each eigenvector, plus relations that hold for the GPU's own outputs (orthonormal
rows, R = B_old B_new^T).  End to end: update, lr_basis_sync with the returned R / B' / A',
fold the block with the new basis, and decode against the oracle of the updated cache."""
import dataclasses

import numpy as np
import pytest

import synth
from oracle import incsvd
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _keys(rng, n, D, decay):
    """Rows with a decaying spectrum in a random orientation."""
    rot = synth.haar_orthonormal(rng, D, D)
    return (rng.standard_normal((n, D)) * decay ** np.arange(D)) @ rot


def _setup(lib, D_heads, r, n0, seed, dtype="f32"):
    import torch
    rng = np.random.default_rng(seed)
    D = D_heads * 128
    K = _keys(rng, n0 + 256, D, 0.985).astype(np.float32).astype(np.float64)
    B0, Z0, S0 = incsvd.initial_basis(K[:n0], r)
    B0 = B0.astype(np.float32)
    desc = lib.make_desc(1, 2 * D_heads, D_heads, 128, r, r, n0 + 300,
                         dtype=lib.LR_F32 if dtype == "f32" else lib.LR_BF16)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()
    c = lib.lr_cache_create(desc, dev(B0.T), dev(B0), dev(B0.T), dev(B0))
    return c, K, B0, S0, D, dev


def _update(lib, c, side, blk, S, r, D, dev):
    import torch
    gram = dev(S)
    R = torch.empty((r, r), dtype=torch.float32, device="cuda")
    Bn = torch.empty((r, D), dtype=torch.float32, device="cuda")
    An = torch.empty((D, r), dtype=torch.float32, device="cuda")
    lib.lr_basis_update(c, side, dev(blk), gram, R, Bn, An)
    torch.cuda.synchronize()
    return gram.cpu().numpy().astype(np.float64), R.cpu().numpy().astype(np.float64), \
        Bn.cpu().numpy().astype(np.float64), An.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("D_heads,r,n", [(2, 32, 16), (4, 128, 128), (4, 256, 64), (8, 400, 100), (2, 16, 1)])
def test_update_matches_oracle(lib, D_heads, r, n):
    c, K, B0, S0, D, dev = _setup(lib, D_heads, r, 600, seed=r + n)
    blk = K[600:600 + n]
    S_in = S0.astype(np.float32).astype(np.float64)
    gram, R, Bn, An = _update(lib, c, 0, blk, S_in, r, D, dev)
    want = incsvd.block_update(B0.astype(np.float64), S_in, blk)
    lam = want["lam"][:r]
    # eigenvalues (fp32 output)
    assert np.allclose(np.diag(gram), lam, rtol=2e-6, atol=1e-6 * lam[0])
    assert np.abs(gram - np.diag(np.diag(gram))).max() == 0.0
    # basis rows and sync columns up to a sign per eigenvector
    sg = np.sign(np.sum(Bn * want["B_new"], axis=1))
    assert np.all(sg != 0)
    assert np.abs(Bn - sg[:, None] * want["B_new"]).max() < 2e-5
    assert np.abs(R - want["R"] * sg[None, :]).max() < 2e-5
    # the GPU's own outputs: orthonormal rows, A' = B'^T, R = B_old B'^T
    assert np.abs(Bn @ Bn.T - np.eye(r)).max() < 1e-5
    assert np.array_equal(An, Bn.T)
    assert np.abs(R - B0.astype(np.float64) @ Bn.T).max() < 1e-5
    lib.lr_cache_destroy(c)


def test_update_on_a_bf16_cache(lib):
    """bf16 basis and block: the GPU and the oracle take the same bf16 values (the basis rows
    then orthonormal only to bf16 precision); the new basis comes back in bf16."""
    import torch
    rng = np.random.default_rng(21)
    D_heads, r, n = 4, 64, 48
    D = D_heads * 128
    K = _keys(rng, 700, D, 0.985)
    B0, _, _ = incsvd.initial_basis(K[:600], r)
    B0b = synth.bf16_to_f64(synth.bf16_bits(B0))
    blk = synth.bf16_to_f64(synth.bf16_bits(K[600:600 + n]))
    Z0 = K[:600] @ B0b.T
    S = (Z0.T @ Z0).astype(np.float32).astype(np.float64)
    desc = lib.make_desc(1, 2 * D_heads, D_heads, 128, r, r, 700)
    tob = lambda x: torch.from_numpy(synth.bf16_bits(x).view(np.int16)).view(torch.bfloat16).cuda()
    c = lib.lr_cache_create(desc, tob(B0b.T), tob(B0b), tob(B0b.T), tob(B0b))
    gram = torch.from_numpy(S.astype(np.float32)).cuda()
    R = torch.empty((r, r), dtype=torch.float32, device="cuda")
    Bn = torch.empty((r, D), dtype=torch.bfloat16, device="cuda")
    lib.lr_basis_update(c, 1, tob(blk), gram, R, Bn)
    torch.cuda.synchronize()
    want = incsvd.block_update(B0b, S, blk)
    got = synth.bf16_to_f64(Bn.cpu().view(torch.int16).numpy().view(np.uint16))
    sg = np.sign(np.sum(got * want["B_new"], axis=1))
    # one bf16 rounding of each entry (plus the fp64 differences of the two factorisations)
    assert np.all(np.abs(got - sg[:, None] * want["B_new"]) <= 2.0 ** -8 * np.abs(want["B_new"]) + 1e-6)
    lam = want["lam"][:r]
    assert np.allclose(np.diag(gram.cpu().numpy()), lam, rtol=1e-5, atol=1e-6 * lam[0])
    lib.lr_cache_destroy(c)


def test_block_inside_the_basis_keeps_the_subspace(lib):
    """A block with no component outside the basis: rank-0 residual, orthogonal R, the same
    subspace (the oracle's in-basis case)."""
    c, K, B0, S0, D, dev = _setup(lib, 2, 32, 400, seed=3)
    rng = np.random.default_rng(5)
    blk = (rng.standard_normal((24, 32)) @ B0.astype(np.float64)).astype(np.float32).astype(np.float64)
    gram, R, Bn, _ = _update(lib, c, 0, blk, S0.astype(np.float32).astype(np.float64), 32, D, dev)
    assert np.abs(R.T @ R - np.eye(32)).max() < 1e-5
    P0 = B0.astype(np.float64).T @ B0.astype(np.float64)
    assert np.abs(Bn.T @ Bn - P0).max() < 1e-5
    lib.lr_cache_destroy(c)


def test_update_sync_fold_then_decode_matches_oracle(lib):
    """The iS-KV step on a whole cache: history latents Z = K_hist B^T, a block of new exact
    keys and values, the basis update of both sides, lr_basis_sync (Z <- Z R, new B and A),
    the block folded in with the new encoder (lr_kv_append), then a decode: equal to the
    oracle decode of the oracle's updated state."""
    import torch
    D_heads, r, n0, n = 2, 48, 500, 32
    rng = np.random.default_rng(11)
    D = D_heads * 128
    Kk = _keys(rng, n0 + n, D, 0.98).astype(np.float32).astype(np.float64)
    Kv = _keys(rng, n0 + n, D, 0.98).astype(np.float32).astype(np.float64)
    Bk, Zk, Sk = incsvd.initial_basis(Kk[:n0], r)
    Bv, Zv, Sv = incsvd.initial_basis(Kv[:n0], r)
    f32 = lambda x: np.ascontiguousarray(x, np.float32)
    Bk32, Bv32 = f32(Bk), f32(Bv)
    desc = lib.make_desc(1, 4 * D_heads, D_heads, 128, r, r, n0 + n + 8, dtype=lib.LR_F32)
    dev = lambda x: torch.from_numpy(f32(x)).cuda()
    c = lib.lr_cache_create(desc, dev(Bk32.T), dev(Bk32), dev(Bv32.T), dev(Bv32))
    Zk32 = f32(Kk[:n0] @ Bk32.T.astype(np.float64))
    Zv32 = f32(Kv[:n0] @ Bv32.T.astype(np.float64))
    lib.lr_kv_append_latent(c, torch.from_numpy(Zk32[None]).cuda(), torch.from_numpy(Zv32[None]).cuda())
    outs = []
    for side, (K, Z32, B32) in enumerate(((Kk, Zk32, Bk32), (Kv, Zv32, Bv32))):
        S = Z32.astype(np.float64).T @ Z32.astype(np.float64)
        gram = dev(S)
        R = torch.empty((r, r), dtype=torch.float32, device="cuda")
        Bn = torch.empty((r, D), dtype=torch.float32, device="cuda")
        An = torch.empty((D, r), dtype=torch.float32, device="cuda")
        lib.lr_basis_update(c, side, dev(K[n0:]), gram, R, Bn, An)
        outs.append((R, Bn, An))
        want = incsvd.block_update(B32.astype(np.float64), f32(S).astype(np.float64), K[n0:])
        outs[-1] = outs[-1] + (want,)
    (Rk, Bkn, Akn, wk), (Rv, Bvn, Avn, wv) = outs
    lib.lr_basis_sync(c, Rk, Rv, Bkn, Bvn, Akn, Avn)
    for t in range(n):
        lib.lr_kv_append(c, dev(Kk[n0 + t][None]), dev(Kv[n0 + t][None]))
    torch.cuda.synchronize()
    assert lib.lr_cache_get_len(c)[0] == n0 + n
    # the oracle's updated state (its own signs; Z B is sign-free)
    zk = np.vstack([Zk32.astype(np.float64) @ wk["R"], Kk[n0:] @ wk["B_new"].T])
    zv = np.vstack([Zv32.astype(np.float64) @ wv["R"], Kv[n0:] @ wv["B_new"].T])
    q = (rng.standard_normal((1, 4 * D_heads, 128)) * 0.3).astype(np.float32)
    p = synth.Problem("incsvd", 1, 4 * D_heads, D_heads, 128, r, r, "f32", 0, False, 1e6, 0, n0 + n,
                      f32(wk["B_new"].T), f32(wk["B_new"]), f32(wv["B_new"].T), f32(wv["B_new"]),
                      f32(zk[None]), f32(zv[None]), q)
    ref, ref_lse = H.oracle_decode(p)
    got, lse = H.gpu_decode(lib, p, c)
    H.compare(p, got, ref, lse, ref_lse, tag="update + sync + fold")
    lib.lr_cache_destroy(c)


def test_update_refusals(lib):
    import torch
    c, K, B0, S0, D, dev = _setup(lib, 2, 32, 300, seed=1)
    g = dev(S0)
    R = torch.empty((32, 32), dtype=torch.float32, device="cuda")
    with pytest.raises(lib.LRError) as e:
        lib.lr_basis_update(c, 0, dev(K[:129]), g, R)          # more than 128 rows
    assert e.value.status == lib.LR_ERR_INVALID_ARG
    with pytest.raises(lib.LRError) as e:
        lib.lr_basis_update(c, 2, dev(K[:8]), g, R)            # no such side
    assert e.value.status == lib.LR_ERR_INVALID_ARG
    lib.lr_cache_destroy(c)


def test_update_time(lib):
    """Time of one update at r = 256, D = 512, n = 128 (reported, not asserted beyond a
    generous bound that catches a runaway)."""
    import torch
    c, K, B0, S0, D, dev = _setup(lib, 4, 256, 400, seed=7)
    blk = dev(K[400:528])
    g0 = dev(S0)
    R = torch.empty((256, 256), dtype=torch.float32, device="cuda")
    Bn = torch.empty((256, D), dtype=torch.float32, device="cuda")
    ts = []
    for _ in range(4):
        g = g0.clone()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        lib.lr_basis_update(c, 0, blk, g, R, Bn)
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    print(f"lr_basis_update r=256 D=512 n=128: {min(ts[1:]) * 1000:.0f} us")
    assert min(ts[1:]) < 200.0
    lib.lr_cache_destroy(c)
