"""Step simulator of the windowed low-rank cache (oracle side, fp64 with storage rounding).

iS-KV abstract and method section: the most recent tokens are kept exactly in
a window; older states are folded, one by one as they leave the window, into
bounded-rank latents z = k A; when the low-rank basis is updated, the stored
historical coordinates are synchronised with it so that the history does not
drift.  The pages give no formula for the update, so the reading here is a
rotation of coordinates: Z_hist <- Z_hist R, with the caller installing the
matching new bases (B' = R^T B keeps Z B unchanged for orthogonal R).

Storage model: history latents and window tokens are stored in the cache dtype;
`store` rounds an fp64 value to it (identity for fp32 caches in this oracle is
fp32 rounding).
"""
from __future__ import annotations

from typing import Callable, List, Optional

import numpy as np

from . import attention
from .quant import round_to_bf16


def store_rounding(dtype: str) -> Callable[[np.ndarray], np.ndarray]:
    if dtype == "bf16":
        return round_to_bf16
    if dtype == "f32":
        return lambda x: np.asarray(x, np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(dtype)


class WindowedCacheSim:
    """History latents [B][n][r] + ring of the last `window` exact tokens."""

    def __init__(self, A_k, B_k, A_v, B_v, n_kv_heads: int, window: int, dtype: str = "bf16"):
        self.A_k = np.asarray(A_k, np.float64)
        self.B_k = np.asarray(B_k, np.float64)
        self.A_v = np.asarray(A_v, np.float64)
        self.B_v = np.asarray(B_v, np.float64)
        self.n_kv_heads = n_kv_heads
        self.window = window
        self.store = store_rounding(dtype)
        self.hist_k: Optional[np.ndarray] = None    # [B][n][r] stored values
        self.hist_v: Optional[np.ndarray] = None
        self.win_k: List[np.ndarray] = []           # oldest first, each [B][D]
        self.win_v: List[np.ndarray] = []

    @property
    def length(self) -> int:
        n = 0 if self.hist_k is None else self.hist_k.shape[1]
        return n + len(self.win_k)

    def _push_hist(self, zk: np.ndarray, zv: np.ndarray) -> None:
        zk = zk[:, None, :]
        zv = zv[:, None, :]
        if self.hist_k is None:
            self.hist_k, self.hist_v = zk, zv
        else:
            self.hist_k = np.concatenate([self.hist_k, zk], axis=1)
            self.hist_v = np.concatenate([self.hist_v, zv], axis=1)

    def fill_history(self, zk_stored: np.ndarray, zv_stored: np.ndarray) -> None:
        """Bulk history fill with already-stored latent values (window must be empty)."""
        assert not self.win_k
        self.hist_k = np.asarray(zk_stored, np.float64).copy()
        self.hist_v = np.asarray(zv_stored, np.float64).copy()

    def append(self, k: np.ndarray, v: np.ndarray) -> None:
        """One new token per sequence (k, v [B][D] exact values).  When the window is
        full, its oldest token is folded into the history first: z = store(k_old A)."""
        if self.window > 0 and len(self.win_k) == self.window:
            k_old = self.win_k.pop(0)
            v_old = self.win_v.pop(0)
            self._push_hist(self.store(attention.project_latent(k_old, self.A_k)),
                            self.store(attention.project_latent(v_old, self.A_v)))
        if self.window > 0:
            self.win_k.append(self.store(k))
            self.win_v.append(self.store(v))
        else:
            self._push_hist(self.store(attention.project_latent(k, self.A_k)),
                            self.store(attention.project_latent(v, self.A_v)))

    def sync(self, R_k=None, R_v=None, B_k_new=None, B_v_new=None, A_k_new=None,
             A_v_new=None) -> None:
        """Rotate stored history coordinates and install new bases (each optional)."""
        if R_k is not None and self.hist_k is not None:
            self.hist_k = self.store(self.hist_k @ np.asarray(R_k, np.float64))
        if R_v is not None and self.hist_v is not None:
            self.hist_v = self.store(self.hist_v @ np.asarray(R_v, np.float64))
        if B_k_new is not None:
            self.B_k = np.asarray(B_k_new, np.float64)
        if B_v_new is not None:
            self.B_v = np.asarray(B_v_new, np.float64)
        if A_k_new is not None:
            self.A_k = np.asarray(A_k_new, np.float64)
        if A_v_new is not None:
            self.A_v = np.asarray(A_v_new, np.float64)

    def decode(self, q: np.ndarray, scale: Optional[float] = None, pairs=None):
        Bsz = q.shape[0]
        r_k, r_v = self.B_k.shape[0], self.B_v.shape[0]
        hk = self.hist_k if self.hist_k is not None else np.zeros((Bsz, 0, r_k))
        hv = self.hist_v if self.hist_v is not None else np.zeros((Bsz, 0, r_v))
        wk = np.stack(self.win_k, axis=1) if self.win_k else None
        wv = np.stack(self.win_v, axis=1) if self.win_v else None
        return attention.decode(q, hk, hv, self.B_k, self.B_v, self.n_kv_heads, scale,
                                None, wk, wv, pairs)
