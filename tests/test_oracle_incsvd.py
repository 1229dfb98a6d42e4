"""Pins of the oracle's block-incremental SVD update (oracle/incsvd.py), on the CPU.

The update is checked against what the mathematics fixes, not against itself:
  - Eckart-Young on the stacked matrix M = [Z B; K_blk]: the new basis spans M's leading
    right singular subspace (from numpy's SVD of M written out, a different routine on a
    different matrix than the update's eigen-decomposition of the small Gram matrix), the
    new Gram matrix holds M's leading squared singular values, and the rank-r residual of M
    has the closed-form norm sqrt(sum_{i>r} s_i^2);
  - exactness: keys of total rank <= r are reproduced exactly after any number of folds;
  - invariants: orthonormal new basis rows, the folded block's coordinates equal K_blk B'^T,
    the sync keeps every stored approximation Z B unchanged inside the new subspace;
  - drift: without the sync, the old coordinates read through the new basis are wrong.
A plausible mistake (a dropped term of the Gram matrix, the wrong block of the eigenvectors
as the sync, a missing residual direction) fails at least one of them.
"""
import numpy as np
import pytest

from oracle import incsvd, svd


def _keys(rng, n, D, decay=0.9):
    return rng.standard_normal((n, D)) * decay ** np.arange(D)


@pytest.mark.parametrize("r,W", [(8, 4), (16, 16), (12, 3)])
def test_update_is_the_truncated_svd_of_the_stacked_matrix(r, W):
    rng = np.random.default_rng(r * 100 + W)
    D = 40
    K = _keys(rng, 60 + W, D)
    B, Z, S = incsvd.initial_basis(K[:60], r)
    up = incsvd.block_update(B, S, K[60:])
    M = np.vstack([Z @ B, K[60:]])
    _, s, vt = np.linalg.svd(M, full_matrices=False)
    # same leading subspace (projectors), Gram = leading s^2, Eckart-Young residual
    Pn = up["B_new"].T @ up["B_new"]
    Pm = vt[:r].T @ vt[:r]
    assert np.abs(Pn - Pm).max() < 1e-9
    assert np.allclose(np.diag(up["S_new"]), s[:r] ** 2, rtol=1e-10, atol=1e-10 * s[0] ** 2)
    res = np.linalg.norm(M - M @ Pn, "fro")
    fro, _ = svd.eckart_young(s, r)
    assert abs(res - fro) <= 1e-9 * max(1.0, fro)
    # invariants
    assert np.abs(up["B_new"] @ up["B_new"].T - np.eye(r)).max() < 1e-12
    assert np.abs(up["Z_blk"] - K[60:] @ up["B_new"].T).max() < 1e-10
    assert np.abs(Z @ up["R"] - (Z @ B) @ up["B_new"].T).max() < 1e-10
    # the synced coordinates reproduce the projection of the old approximation
    assert np.abs((Z @ up["R"]) @ up["B_new"] - (Z @ B) @ Pn).max() < 1e-10


def test_low_rank_keys_are_reproduced_exactly_after_many_folds():
    rng = np.random.default_rng(5)
    D, r, true_rank = 48, 10, 7
    basis = np.linalg.qr(rng.standard_normal((D, true_rank)))[0].T
    K = rng.standard_normal((300, true_rank)) @ basis
    B, Z = incsvd.fold_blocks(K, r, 32, 16)
    assert np.abs(Z @ B - K).max() < 1e-10
    assert np.abs(B @ B.T - np.eye(r)).max() < 1e-12


def test_folded_history_matches_one_shot_svd_when_blocks_stay_in_rank():
    """Keys whose whole history has rank <= r: the folded basis spans the same subspace as
    the one-shot SVD of all keys (Eckart-Young with zero tail)."""
    rng = np.random.default_rng(11)
    D, r = 32, 6
    basis = np.linalg.qr(rng.standard_normal((D, r)))[0].T
    K = rng.standard_normal((200, r)) @ basis
    B, _ = incsvd.fold_blocks(K, r, 20, 8)
    _, _, vt = np.linalg.svd(K, full_matrices=False)
    assert np.abs(B.T @ B - vt[:r].T @ vt[:r]).max() < 1e-10


def test_block_inside_the_basis_gives_an_orthogonal_sync():
    """A block that adds no direction outside the basis: R is orthogonal (the update only
    rotates inside the subspace) and the sync keeps Z B exactly."""
    rng = np.random.default_rng(2)
    D, r = 24, 8
    K0 = _keys(rng, 40, D)
    B, Z, S = incsvd.initial_basis(K0, r)
    blk = rng.standard_normal((5, r)) @ B
    up = incsvd.block_update(B, S, blk)
    assert np.abs(up["R"].T @ up["R"] - np.eye(r)).max() < 1e-10
    assert np.abs((Z @ up["R"]) @ up["B_new"] - Z @ B).max() < 1e-10


def test_skipping_the_sync_drifts():
    """Old coordinates read through the new basis without the sync misrepresent the
    history (the drift the iS-KV abstract reports for unsynchronised coordinates)."""
    rng = np.random.default_rng(9)
    D, r = 40, 8
    K = _keys(rng, 80, D, decay=0.97)
    B, Z, S = incsvd.initial_basis(K[:60], r)
    up = incsvd.block_update(B, S, K[60:] * 3.0)
    synced = (Z @ up["R"]) @ up["B_new"]
    stale = Z @ up["B_new"]
    ref = (Z @ B) @ (up["B_new"].T @ up["B_new"])
    assert np.abs(synced - ref).max() < 1e-10
    assert np.linalg.norm(stale - ref) > 0.1 * np.linalg.norm(ref)


def test_planted_gram_mistake_is_caught():
    """The pin above fails for an update that forgets the history's Gram term S."""
    rng = np.random.default_rng(4)
    D, r, W = 30, 6, 4
    K = _keys(rng, 40 + W, D)
    B, Z, S = incsvd.initial_basis(K[:40], r)
    bad = incsvd.block_update(B, np.zeros_like(S), K[40:])
    M = np.vstack([Z @ B, K[40:]])
    _, _, vt = np.linalg.svd(M, full_matrices=False)
    assert np.abs(bad["B_new"].T @ bad["B_new"] - vt[:r].T @ vt[:r]).max() > 1e-3
