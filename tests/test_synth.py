"""CPU checks of the seeded input generators (`synth/`): the properties the input recipe
states — the stand-in rank allocation, the bases' structure, the latents' spectrum, the
exact fold of the hybrid's window tokens, the sync rotations, seed determinism — hold for
the arrays the tests and the bench draw."""
import numpy as np
import pytest

import synth


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_rank_allocation_invariants(seed):
    """Multiples of 16 in [128, 448] with the mean exactly 256, reproducible per seed."""
    r = synth.global_rank_allocation(28, synth.rng_for("qwen32k", "ranks_k", seed))
    again = synth.global_rank_allocation(28, synth.rng_for("qwen32k", "ranks_k", seed))
    assert np.array_equal(r, again)
    assert np.all(r % 16 == 0) and r.min() >= 128 and r.max() <= 448
    assert r.sum() == 28 * 256
    assert r.max() - r.min() >= 160                 # the transfers spread the ranks


def test_qwen32k_layer_ranks_named_by_the_tests():
    """The per-layer (r_k, r_v) that the parity tests cite for seed 0."""
    ranks = synth.qwen32k_ranks(0)
    assert len(ranks) == 28
    assert ranks[0] == (256, 384) and ranks[5] == (128, 128) and ranks[4] == (400, 224)
    assert ranks[11] == (448, 256) and ranks[12] == (192, 448)
    rk, rv = np.array(ranks).T
    assert rk.sum() == rv.sum() == 28 * 256


@pytest.mark.parametrize("rows, cols", [(32, 64), (256, 512), (64, 64)])
def test_haar_rows_are_orthonormal(rows, cols):
    q = synth.haar_orthonormal(synth.rng_for("t", "haar", 0), rows, cols)
    assert q.shape == (rows, cols)
    assert np.max(np.abs(q @ q.T - np.eye(rows))) < 1e-12


def test_sync_rotation_is_orthogonal_and_seeded():
    R = synth.sync_rotation(0, 3, 256)
    assert np.max(np.abs(R @ R.T - np.eye(256))) < 1e-12
    assert np.array_equal(R, synth.sync_rotation(0, 3, 256))
    assert not np.allclose(R, synth.sync_rotation(0, 4, 256))
    assert not np.allclose(R, synth.sync_rotation(0, 3, 256, "v"))


def test_qwen_bases_make_a_projector():
    """B has orthonormal rows scaled by 1/sqrt(r) and A = r B^T, so A B projects onto the
    row space of B (up to the bf16 storage of both)."""
    p = synth.make_qwen("qwen4k", seed=0, batch=1, length=1, rank=256)
    A, B = synth.bf16_to_f64(p.A_k), synth.bf16_to_f64(p.B_k)
    r = p.rank_k
    assert np.max(np.abs(B @ B.T * r - np.eye(r))) < 5e-3            # bf16 rows (observed 8e-4)
    assert np.max(np.abs(A - r * B.T)) <= 2.0 ** -8 * np.max(np.abs(A))
    P = A @ B
    assert np.max(np.abs(P @ P - P)) < 5e-3                          # idempotent up to rounding


def test_latent_spectrum():
    """Latents N(0,1) x i^-0.7 per rank coordinate."""
    p = synth.make_qwen("qwen4k", seed=0, batch=4, length=4096, rank=256)
    std = p.z_k.reshape(-1, 256).astype(np.float64).std(axis=0)
    ratio = std / synth.spectrum(256, 0.7)
    assert np.all(np.abs(ratio - 1.0) < 0.03), (ratio.min(), ratio.max())


def test_hybrid_token_folds_exactly():
    """Window tokens are k = (g x sigma) B_k, so the fold k A_k with A_k = r B_k^T returns
    g x sigma exactly (fp64, unrounded bases)."""
    r, D, B = 256, 1024, 3
    Bk = synth.haar_orthonormal(synth.rng_for("t", "Bk", 0), r, D) / np.sqrt(r)
    Bv = synth.haar_orthonormal(synth.rng_for("t", "Bv", 0), r, D) / np.sqrt(r)
    k, v = synth.hybrid_token("hybrid", 0, 7, B, D, Bk, Bv)
    rng = synth.rng_for("hybrid", "tok/7", 0)
    gk = rng.standard_normal((B, r)) * synth.spectrum(r, 0.7)[None]
    gv = rng.standard_normal((B, r)) * synth.spectrum(r, 0.7)[None]
    assert np.max(np.abs(k @ (r * Bk.T) - gk)) < 1e-12
    assert np.max(np.abs(v @ (r * Bv.T) - gv)) < 1e-12


def test_tiny_keys_have_the_stated_spectrum():
    """tiny: K = G diag(i^-0.8) Q^T with Gaussian G (256 x 64), so its singular values are
    sqrt(T) i^-0.8 up to the sampling spread of G; A, B are its top-32 right singular
    vectors (orthonormal rows)."""
    p = synth.make_tiny(0)
    K = p.extra["K"][0].astype(np.float64)
    s = np.linalg.svd(K, compute_uv=False)
    ratio = s / (np.sqrt(K.shape[0]) * synth.spectrum(K.shape[1], 0.8))
    assert np.all((ratio > 0.6) & (ratio < 1.4)), (ratio.min(), ratio.max())
    B = p.B_k.astype(np.float64)
    assert np.max(np.abs(B @ B.T - np.eye(p.rank_k))) < 1e-6


def test_draws_are_keyed_by_workload_tensor_and_seed():
    a = synth.rng_for("qwen4k", "q/0", 0).standard_normal(8)
    assert np.array_equal(a, synth.rng_for("qwen4k", "q/0", 0).standard_normal(8))
    assert not np.allclose(a, synth.rng_for("qwen4k", "q/0", 1).standard_normal(8))
    assert not np.allclose(a, synth.rng_for("qwen4k", "q/1", 0).standard_normal(8))
    assert not np.allclose(a, synth.rng_for("qwen16k", "q/0", 0).standard_normal(8))
