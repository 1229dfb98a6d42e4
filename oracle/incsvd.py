"""Block-incremental SVD update of the latent basis (oracle side, fp64) — TEST
INFRASTRUCTURE ONLY, like the rest of `oracle/`.

iS-KV (title: "Online Low-Rank KV Cache Compression via Block-Incremental SVD"; method
section, technical framework and key innovation: a dynamically updated low-rank basis,
kept current by an incremental SVD update, with the historical coordinates synchronised
to it).  The pages name the technique but give no formula, so this module takes the
textbook block update of a truncated SVD (the plainest reading), in the cache's own terms:

  state     B [r][D]  orthonormal basis rows; the stored history coordinates are
                      Z = K_hist B^T ([n][r]), and S = Z^T Z ([r][r]) is their Gram matrix
                      (diagonal when B is the SVD basis of the history)
  block     K_blk [W][D], the tokens folded out of the window
  step 1    Y = K_blk B^T                 coordinates of the block in the current basis
  step 2    P = K_blk - Y B = Rp^T Q^T    the residual outside the basis, with Q [D][W]
                                          orthonormal columns orthogonal to B's rows
  step 3    C = [[Z, 0], [Y, Rp^T]] is the matrix [Z B; K_blk] in the basis [B; Q^T];
            its Gram matrix needs only S:  G = [[S + Y^T Y, Y^T Rp^T], [Rp Y, Rp Rp^T]]
  step 4    the r leading eigenvectors V ([r + W][r]) of G (eigenvalues lam, descending;
            W shrinks to the number of new directions when the block has fewer)
  result    B' = V^T [B; Q^T]      new basis (rows orthonormal)
            R  = V[:r, :]          sync rotation: stored history Z <- Z R  (= Z B B'^T)
            Z_blk = [Y, Rp^T] V    coordinates of the folded block (= K_blk B'^T)
            S' = diag(lam[:r])     Gram matrix of the updated coordinates

B' spans the leading right singular subspace of [Z B; K_blk], so by the Eckart-Young
theorem the update keeps the best rank-r approximation of the current approximation stacked
with the new block.  (R is the top block of an orthogonal matrix, orthogonal only when the
block adds nothing outside the old basis.)
"""
from __future__ import annotations

import numpy as np


def initial_basis(K0: np.ndarray, r: int):
    """The state after the first block: the rank-r truncated SVD of K0 ([n][D]).
    Returns (B [r][D], Z = K0 B^T [n][r], S = Z^T Z [r][r])."""
    K0 = np.asarray(K0, np.float64)
    _, s, vt = np.linalg.svd(K0, full_matrices=False)
    B = vt[:r, :].copy()
    Z = K0 @ B.T
    return B, Z, Z.T @ Z


def _residual_basis(P: np.ndarray, B: np.ndarray):
    """Q [D][W'] with orthonormal columns orthogonal to the rows of B, spanning the rows of
    P, and Rp [W'][W] with P = Rp^T Q^T.  Householder QR of P^T; its columns are projected
    once more off the basis and orthonormalised by an SVD that drops any column the
    projection removed (W' <= W when the block adds fewer than W new directions), then
    projected and orthonormalised a second time (two passes of Gram-Schmidt)."""
    Q, _ = np.linalg.qr(P.T)
    Q = Q - B.T @ (B @ Q)
    U, sv, _ = np.linalg.svd(Q, full_matrices=False)
    Q = U[:, sv > 1e-6]
    Q = Q - B.T @ (B @ Q)            # second pass: orthogonal to B to working precision
    Q, _ = np.linalg.qr(Q)
    Rp = Q.T @ P.T
    return Q, Rp


def block_update(B: np.ndarray, S: np.ndarray, K_blk: np.ndarray):
    """One block-incremental update (steps 1-4 above).  Returns a dict with B_new, R,
    Z_blk, S_new and lam (every eigenvalue of G, descending)."""
    B = np.asarray(B, np.float64)
    S = np.asarray(S, np.float64)
    K_blk = np.asarray(K_blk, np.float64)
    r = B.shape[0]
    Y = K_blk @ B.T                                       # step 1
    P = K_blk - Y @ B                                     # step 2
    Q, Rp = _residual_basis(P, B)
    W = Q.shape[1]
    G = np.zeros((r + W, r + W))                          # step 3
    G[:r, :r] = S + Y.T @ Y
    G[:r, r:] = Y.T @ Rp.T
    G[r:, :r] = Rp @ Y
    G[r:, r:] = Rp @ Rp.T
    G = 0.5 * (G + G.T)
    lam, vecs = np.linalg.eigh(G)                         # step 4 (ascending)
    order = np.argsort(lam)[::-1]
    lam = lam[order]
    V = vecs[:, order[:r]]
    B_new = V.T @ np.vstack([B, Q.T])
    R = V[:r, :].copy()
    Z_blk = np.hstack([Y, Rp.T]) @ V
    return {"B_new": B_new, "R": R, "Z_blk": Z_blk, "S_new": np.diag(lam[:r]), "lam": lam}


def fold_blocks(K: np.ndarray, r: int, n0: int, W: int):
    """Run the update over a whole key matrix: the first n0 rows give the initial basis, then
    blocks of W rows are folded one after another, each time syncing the stored history.
    Returns (B, Z) with Z the synced coordinates of every row ([n][r])."""
    K = np.asarray(K, np.float64)
    B, Z, S = initial_basis(K[:n0], r)
    for s0 in range(n0, K.shape[0], W):
        up = block_update(B, S, K[s0:s0 + W])
        Z = np.vstack([Z @ up["R"], up["Z_blk"]])
        B, S = up["B_new"], up["S_new"]
    return B, Z
