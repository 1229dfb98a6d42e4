"""Decode attention over a stored low-rank cache, by its plain definition (fp64).

TraceKV abstract: the cache holds low-dimensional latents of the KV states;
keys and values are recovered through shared bases, K = Z_k B_k and
V = Z_v B_v.  The digest's Perspective section fixes the decode workload
(Qwen2.5-VL-7B, batch 16, context 4K-32K).  The iS-KV abstract adds an exact
recent window kept next to the low-rank history.

The oracle does not use the latent-space shortcut the GPU path takes; it
reconstructs every key and value and runs textbook softmax attention:

  K^_cat = Z^_k B_k,  V^_cat = Z^_v B_v       (Z^ = stored or dequantised latents)
  head h of a token = columns [h d, (h+1) d) of the concatenated KV projection
  query head j reads KV head h(j) = j // (Hq / Hkv)          (contiguous GQA groups)
  keys compressed before RoPE are rotated (rotate-half, theta) at their position
  window tokens (exact K, V) follow the history tokens
  logits_t = s * q_j . k_t,   w = softmax(logits),   o_j = sum_t w_t v_t
  lse_j = log sum_t exp(logits_t)                   (natural log)
"""
from __future__ import annotations

from typing import Iterable, Optional, Sequence, Tuple

import numpy as np


def reconstruct(Z: np.ndarray, B: np.ndarray) -> np.ndarray:
    """K^ = Z B  ([T][r] x [r][D] -> [T][D]), fp64."""
    return np.asarray(Z, dtype=np.float64) @ np.asarray(B, dtype=np.float64)


def rope_rotate_half(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half RoPE of rows x[t] ([T][d]) at absolute positions (fp64 angles).

    omega_i = theta^(-2i/d) for i < d/2;
    x'[i]       = x[i] cos(t omega_i) - x[i + d/2] sin(t omega_i)
    x'[i + d/2] = x[i + d/2] cos(t omega_i) + x[i] sin(t omega_i)
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    i = np.arange(half, dtype=np.float64)
    omega = float(theta) ** (-2.0 * i / d)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * omega[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[:, :half], x[:, half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=1)


def softmax_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """Textbook single-query attention with max subtraction.
    q [d], K [T][d], V [T][d] -> (o [d], lse, weights [T])."""
    logits = scale * (np.asarray(K, np.float64) @ np.asarray(q, np.float64))
    m = logits.max()
    e = np.exp(logits - m)
    l = e.sum()
    w = e / l
    o = w @ np.asarray(V, np.float64)
    return o, m + np.log(l), w


def kv_head_of(j: int, n_q_heads: int, n_kv_heads: int) -> int:
    return j // (n_q_heads // n_kv_heads)


def decode(q: np.ndarray, Zk: np.ndarray, Zv: np.ndarray, Bk: np.ndarray, Bv: np.ndarray,
           n_kv_heads: int, scale: Optional[float] = None, rope_theta: Optional[float] = None,
           win_k: Optional[np.ndarray] = None, win_v: Optional[np.ndarray] = None,
           pairs: Optional[Iterable[Tuple[int, int]]] = None):
    """Decode attention of one step over a stored cache.

    q      [B][Hq][d]      query (already rotated when keys carry RoPE)
    Zk, Zv [B][T][r]       stored latent values (dequantised / bf16 values, fp64)
    Bk, Bv [r][Hkv*d]      bases
    win_k, win_v [B][W][Hkv*d] exact window tokens following the history, or None
    rope_theta             if set, reconstructed history keys are rotated at 0..T-1
    pairs                  (b, j) outputs to compute; default all.
    Returns (out [B][Hq][d], lse [B][Hq]); entries not in `pairs` are NaN.
    """
    q = np.asarray(q, dtype=np.float64)
    Bsz, Hq, d = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    if rope_theta is not None and win_k is not None and np.asarray(win_k).shape[1] > 0:
        raise ValueError("RoPE-in-kernel caches carry no exact window")
    out = np.full((Bsz, Hq, d), np.nan)
    lse = np.full((Bsz, Hq), np.nan)
    if pairs is None:
        pairs = [(b, j) for b in range(Bsz) for j in range(Hq)]
    Bk = np.asarray(Bk, np.float64)
    Bv = np.asarray(Bv, np.float64)
    cache = {}
    for b, j in pairs:
        h = kv_head_of(j, Hq, n_kv_heads)
        key = (b, h)
        if key not in cache:
            cols = slice(h * d, (h + 1) * d)
            Kh = reconstruct(Zk[b], Bk[:, cols])
            Vh = reconstruct(Zv[b], Bv[:, cols])
            if rope_theta is not None:
                Kh = rope_rotate_half(Kh, np.arange(Kh.shape[0]), rope_theta)
            if win_k is not None:
                Kh = np.concatenate([Kh, np.asarray(win_k[b], np.float64)[:, cols]], axis=0)
                Vh = np.concatenate([Vh, np.asarray(win_v[b], np.float64)[:, cols]], axis=0)
            cache = {key: (Kh, Vh)}          # keep one head resident
        Kh, Vh = cache[key]
        o, l, _ = softmax_attention(q[b, j], Kh, Vh, scale)
        out[b, j] = o
        lse[b, j] = l
    return out, lse


def project_latent(x: np.ndarray, A: np.ndarray) -> np.ndarray:
    """z = x A for new tokens ([..., D] x [D][r]), fp64 (the append projection)."""
    return np.asarray(x, np.float64) @ np.asarray(A, np.float64)


def sample_pairs(batch: int, n_q_heads: int, count: int, seed: int = 0) -> Sequence[Tuple[int, int]]:
    """A deterministic spread of (b, j) output coordinates for full-size spot checks:
    always the first and last head of the first and last sequence, plus seeded picks."""
    rng = np.random.default_rng(seed)
    fixed = {(0, 0), (0, n_q_heads - 1), (batch - 1, 0), (batch - 1, n_q_heads - 1)}
    picks = set(fixed)
    while len(picks) < min(count, batch * n_q_heads):
        picks.add((int(rng.integers(batch)), int(rng.integers(n_q_heads))))
    return sorted(picks)
