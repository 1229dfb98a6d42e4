"""Seeded synthetic inputs for the low-rank KV-cache decode path.

This module is shared by the tests, the oracle-side checks and the bench.  It
holds no arithmetic of the method itself: only random draws, decaying spectra,
Haar-random orthonormal frames, the stand-in rank allocation, and rounding of
the drawn values to the storage dtype.  Everything is fp64 until the final
rounding, and every draw is keyed by (workload, tensor name, seed) so each
tensor is reproducible on its own.

Workloads (sizes follow the TraceKV latency setup, "Perspective" section of the
ai4snews digest: Qwen2.5-VL-7B at batch 16, 4K-32K context; the hybrid follows
the iS-KV abstract: exact recent window plus low-rank history on Qwen3-8B):

  tiny      fp32, B=1, Hq=2, Hkv=1, d=64, T=256, r=32; K, V = G diag(i^-0.8) Q^T,
            A and B from the truncated SVD of K and of V.
  qwen4k    bf16, B=16, Hq=28, Hkv=4, d=128, T=4096, r=256; latents N(0,1)*i^-0.7.
  qwen16k   as qwen4k at r=352, int4 group-32 latents, T=16384.
  qwen32k   28 layers, T=32768, int4, per-layer ranks in [128,448] (mean 256),
            keys compressed before RoPE (theta 1e6).
  hybrid    bf16, B=8, Hq=32, Hkv=8, d=128, T=32768 = 32640 history (r=256)
            + 128-token exact window; seeded Haar 256x256 rotations for sync.
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Dict, List, Optional

import numpy as np

# ----------------------------------------------------------------------------
# dtype helpers (storage rounding only)
# ----------------------------------------------------------------------------


def bf16_bits(x) -> np.ndarray:
    """Round to bfloat16 (round-to-nearest-even) and return the uint16 bit patterns.

    fp64 input is first rounded to fp32 (RNE), then to bf16 (RNE).  Finite inputs only.
    """
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    return r


def bf16_to_f64(bits) -> np.ndarray:
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_bf16(x) -> np.ndarray:
    """fp64 value of the bf16 rounding of x."""
    return bf16_to_f64(bf16_bits(x))


# ----------------------------------------------------------------------------
# seeded generators
# ----------------------------------------------------------------------------


def rng_for(workload: str, tensor: str, seed: int = 0) -> np.random.Generator:
    """Independent PCG64 stream per (workload, tensor, seed)."""
    h = hashlib.sha256(f"{workload}/{tensor}".encode()).digest()
    key = [int.from_bytes(h[i:i + 4], "little") for i in range(0, 16, 4)]
    return np.random.default_rng(np.random.SeedSequence([seed] + key))


def spectrum(n: int, power: float) -> np.ndarray:
    """sigma_i = i^-power for i = 1..n."""
    return np.arange(1, n + 1, dtype=np.float64) ** (-power)


def haar_orthonormal(rng: np.random.Generator, rows: int, cols: int) -> np.ndarray:
    """A rows x cols matrix with orthonormal rows (rows <= cols), Haar distributed.

    QR of a cols x rows Gaussian matrix with the sign of diag(R) folded into Q.
    """
    assert rows <= cols
    g = rng.standard_normal((cols, rows))
    q, r = np.linalg.qr(g)
    q = q * np.sign(np.diag(r))[None, :]
    return np.ascontiguousarray(q.T)


def haar_orthogonal(rng: np.random.Generator, n: int) -> np.ndarray:
    return haar_orthonormal(rng, n, n)


def global_rank_allocation(n_layers: int, rng: np.random.Generator, mean: int = 256,
                           lo: int = 128, hi: int = 448, step: int = 16,
                           moves: int = 10000) -> np.ndarray:
    """Stand-in for TraceKV's global rank allocation (abstract; Synopsis of the digest).

    The pages give no algorithm, so ranks start at `mean` and take `moves` seeded
    transfers of `step` from a random layer to another while both stay in [lo, hi].
    The sum, hence the mean, is preserved exactly.
    """
    ranks = np.full(n_layers, mean, dtype=np.int64)
    for _ in range(moves):
        i, j = rng.integers(0, n_layers, size=2)
        if i == j:
            continue
        if ranks[i] - step >= lo and ranks[j] + step <= hi:
            ranks[i] -= step
            ranks[j] += step
    return ranks


# ----------------------------------------------------------------------------
# problem container
# ----------------------------------------------------------------------------


@dataclasses.dataclass
class Problem:
    """One layer's decode problem.

    Stored tensors are given in their storage form: fp32 arrays for dtype
    "f32", uint16 bf16 bit patterns for dtype "bf16".  Latent tensors z_k/z_v
    are fp32 (the values handed to the latent fill / quantiser).
    """
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    rank_k: int
    rank_v: int
    dtype: str                   # "f32" | "bf16"
    quant_bits: int              # 0 | 4
    rope: bool
    rope_theta: float
    window: int
    hist_len: int                # tokens held as latents
    A_k: np.ndarray              # [D][r_k] storage dtype
    B_k: np.ndarray              # [r_k][D]
    A_v: np.ndarray
    B_v: np.ndarray
    z_k: np.ndarray              # [B][hist_len][r_k] fp32
    z_v: np.ndarray
    q: np.ndarray                # [B][Hq][d] storage dtype
    win_k: Optional[np.ndarray] = None   # [B][win][D] storage dtype (exact window tokens)
    win_v: Optional[np.ndarray] = None
    extra: Dict[str, np.ndarray] = dataclasses.field(default_factory=dict)

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def win_len(self) -> int:
        return 0 if self.win_k is None else self.win_k.shape[1]

    @property
    def length(self) -> int:
        return self.hist_len + self.win_len

    def to_f64(self, x: np.ndarray) -> np.ndarray:
        """fp64 value of a stored tensor."""
        if self.dtype == "bf16":
            return bf16_to_f64(x)
        return np.asarray(x, dtype=np.float64)

    def store(self, x: np.ndarray) -> np.ndarray:
        """Round fp64 values to this problem's storage form."""
        if self.dtype == "bf16":
            return bf16_bits(x)
        return np.asarray(x, dtype=np.float32)


def _store(dtype: str, x: np.ndarray) -> np.ndarray:
    return bf16_bits(x) if dtype == "bf16" else np.asarray(x, dtype=np.float32)


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------


def make_tiny(seed: int = 0, length: int = 256, sharp: float = 1.0) -> Problem:
    """fp32 correctness case: K, V = G diag(i^-0.8) Q^T; A, B from the truncated SVD."""
    name = "tiny"
    B, Hq, Hkv, d, r = 1, 2, 1, 64, 32
    D = Hkv * d
    sig = spectrum(D, 0.8)
    out = {}
    for nm in ("k", "v"):
        g = rng_for(name, f"{nm}_gauss", seed).standard_normal((length, D))
        Q = haar_orthogonal(rng_for(name, f"{nm}_frame", seed), D)
        X = (g * sig[None, :]) @ Q
        # truncated SVD of the generated matrix (input synthesis, a library routine)
        _, _, vt = np.linalg.svd(X, full_matrices=False)
        Bm = vt[:r, :]                       # [r][D], orthonormal rows
        Am = Bm.T.copy()                     # [D][r]
        out[nm] = (X, Am, Bm)
    Kx, A_k, B_k = out["k"]
    Vx, A_v, B_v = out["v"]
    A_k32, B_k32 = A_k.astype(np.float32), B_k.astype(np.float32)
    A_v32, B_v32 = A_v.astype(np.float32), B_v.astype(np.float32)
    # latents are the projections through the stored fp32 A, in fp64, rounded to fp32
    z_k = (Kx @ A_k32.astype(np.float64)).astype(np.float32)[None]
    z_v = (Vx @ A_v32.astype(np.float64)).astype(np.float32)[None]
    q = rng_for(name, "q", seed).standard_normal((B, Hq, d)) * sharp
    p = Problem(name, B, Hq, Hkv, d, r, r, "f32", 0, False, 1e6, 0, length,
                A_k32, B_k32, A_v32, B_v32, z_k, z_v, q.astype(np.float32))
    p.extra["K"] = Kx[None].astype(np.float32)
    p.extra["V"] = Vx[None].astype(np.float32)
    return p


def _qwen_bases(name: str, seed: int, r_k: int, r_v: int, D: int, dtype: str, layer: int = 0):
    """B: Haar orthonormal rows scaled by 1/sqrt(r); A = r * B^T so that A B is the
    orthogonal projector onto the row space of B."""
    Bk = haar_orthonormal(rng_for(name, f"B_k/{layer}", seed), r_k, D) / np.sqrt(r_k)
    Bv = haar_orthonormal(rng_for(name, f"B_v/{layer}", seed), r_v, D) / np.sqrt(r_v)
    Ak = r_k * Bk.T
    Av = r_v * Bv.T
    return _store(dtype, Ak), _store(dtype, Bk), _store(dtype, Av), _store(dtype, Bv)


def grouped_bases(name: str, seed: int, g: int, r: int, D: int, dtype: str = "bf16"):
    """Per-group bases of a cache with g latent groups of rank r: B_i with Haar orthonormal
    rows scaled by 1/sqrt(r) over the group's D/g coordinates, A_i = r B_i^T.  Returns the
    compact forms (A [g][D/g][r], B [g][r][D/g], for K then V) and the block-diagonal
    B_k, B_v ([g r][D], fp64) they stand for."""
    Dg = D // g
    out = []
    for side in ("k", "v"):
        rng = rng_for(name, f"B_{side}/groups{g}", seed)
        Bs = np.stack([haar_orthonormal(rng, r, Dg) / np.sqrt(r) for _ in range(g)])
        full = np.zeros((g * r, D))
        for i in range(g):
            full[i * r:(i + 1) * r, i * Dg:(i + 1) * Dg] = Bs[i]
        out.append((_store(dtype, r * Bs.transpose(0, 2, 1)), _store(dtype, Bs), full))
    (Ak, Bk, Bk_full), (Av, Bv, Bv_full) = out
    return Ak, Bk, Av, Bv, Bk_full, Bv_full


def _latents(name: str, tensor: str, seed: int, B: int, T: int, r: int, power: float) -> np.ndarray:
    g = rng_for(name, tensor, seed).standard_normal((B, T, r))
    return (g * spectrum(r, power)[None, None, :]).astype(np.float32)


def make_qwen(name: str = "qwen4k", seed: int = 0, batch: int = 16, length: int = 4096,
              rank: int = 256, quant_bits: int = 0, rope: bool = False,
              n_q_heads: int = 28, n_kv_heads: int = 4, head_dim: int = 128,
              sharp: float = 1.0, layer: int = 0, rank_v: Optional[int] = None) -> Problem:
    """Qwen2.5-VL-7B-shaped single layer: latents N(0,1) * i^-0.7, Haar bases / sqrt(r),
    q ~ N(0,1)/sqrt(128) (times `sharp`)."""
    r_k = rank
    r_v = rank if rank_v is None else rank_v
    D = n_kv_heads * head_dim
    A_k, B_k, A_v, B_v = _qwen_bases(name, seed, r_k, r_v, D, "bf16", layer)
    z_k = _latents(name, f"z_k/{layer}", seed, batch, length, r_k, 0.7)
    z_v = _latents(name, f"z_v/{layer}", seed, batch, length, r_v, 0.7)
    q = rng_for(name, f"q/{layer}", seed).standard_normal((batch, n_q_heads, head_dim))
    q = q / np.sqrt(128.0) * sharp
    return Problem(name, batch, n_q_heads, n_kv_heads, head_dim, r_k, r_v, "bf16",
                   quant_bits, rope, 1e6, 0, length, A_k, B_k, A_v, B_v, z_k, z_v,
                   bf16_bits(q))


def qwen32k_ranks(seed: int = 0, n_layers: int = 28):
    """Per-layer (r_k, r_v) of the 28-layer int4 workload."""
    rk = global_rank_allocation(n_layers, rng_for("qwen32k", "ranks_k", seed))
    rv = global_rank_allocation(n_layers, rng_for("qwen32k", "ranks_v", seed))
    return [(int(a), int(b)) for a, b in zip(rk, rv)]


def make_qwen32k_layer(layer: int, seed: int = 0, batch: int = 16, length: int = 32768,
                       rope: bool = True, sharp: float = 1.0) -> Problem:
    rk, rv = qwen32k_ranks(seed)[layer]
    return make_qwen("qwen32k", seed, batch, length, rk, 4, rope, sharp=sharp,
                     layer=layer, rank_v=rv)


def hybrid_token(name: str, seed: int, step: int, B: int, D: int, Bk: np.ndarray,
                 Bv: np.ndarray, noise: float = 0.0):
    """One appended token per sequence: k = (g * sigma) B_k (+ relative noise), so that its
    fold k A_k = g * sigma has the same law as the stored history latents."""
    rk, rv = Bk.shape[0], Bv.shape[0]
    rng = rng_for(name, f"tok/{step}", seed)
    gk = rng.standard_normal((B, rk)) * spectrum(rk, 0.7)[None]
    gv = rng.standard_normal((B, rv)) * spectrum(rv, 0.7)[None]
    k = gk @ Bk
    v = gv @ Bv
    if noise:
        k = k + noise * rng.standard_normal((B, D)) * np.abs(k).mean()
        v = v + noise * rng.standard_normal((B, D)) * np.abs(v).mean()
    return k, v


def make_hybrid(seed: int = 0, batch: int = 8, hist_len: int = 32640, window: int = 128,
                win_len: Optional[int] = None, rank: int = 256, n_q_heads: int = 32,
                n_kv_heads: int = 8, head_dim: int = 128, sharp: float = 1.0) -> Problem:
    """Qwen3-8B-shaped iS-KV hybrid: exact bf16 window plus bf16 low-rank history."""
    name = "hybrid"
    D = n_kv_heads * head_dim
    A_k, B_k, A_v, B_v = _qwen_bases(name, seed, rank, rank, D, "bf16")
    z_k = _latents(name, "z_k", seed, batch, hist_len, rank, 0.7)
    z_v = _latents(name, "z_v", seed, batch, hist_len, rank, 0.7)
    wl = window if win_len is None else win_len
    Bk64, Bv64 = bf16_to_f64(B_k), bf16_to_f64(B_v)
    ks, vs = [], []
    for t in range(wl):
        k, v = hybrid_token(name, seed, hist_len + t, batch, D, Bk64, Bv64, noise=1e-2)
        ks.append(k)
        vs.append(v)
    win_k = bf16_bits(np.stack(ks, axis=1)) if wl else np.zeros((batch, 0, D), np.uint16)
    win_v = bf16_bits(np.stack(vs, axis=1)) if wl else np.zeros((batch, 0, D), np.uint16)
    q = rng_for(name, "q", seed).standard_normal((batch, n_q_heads, head_dim))
    q = q / np.sqrt(128.0) * sharp
    return Problem(name, batch, n_q_heads, n_kv_heads, head_dim, rank, rank, "bf16", 0,
                   False, 1e6, window, hist_len, A_k, B_k, A_v, B_v, z_k, z_v,
                   bf16_bits(q), win_k, win_v)


def sync_rotation(seed: int, event: int, r: int, which: str = "k") -> np.ndarray:
    """Seeded Haar r x r orthogonal matrix for the `event`-th basis sync (stand-in for the
    block-incremental SVD basis update of iS-KV)."""
    return haar_orthogonal(rng_for("hybrid", f"R_{which}/{event}", seed), r)


def small_variant(kind: str, seed: int = 0, **kw) -> Problem:
    """Reduced-size variants of each workload for parity tests (several tiles plus a
    ragged tail)."""
    if kind == "tiny":
        return make_tiny(seed, **kw)
    if kind == "qwen4k":
        kw.setdefault("batch", 2)
        kw.setdefault("length", 1000)
        return make_qwen("qwen4k", seed, **kw)
    if kind == "qwen16k":
        kw.setdefault("batch", 2)
        kw.setdefault("length", 1000)
        kw.setdefault("rank", 352)
        kw.setdefault("quant_bits", 4)
        return make_qwen("qwen16k", seed, **kw)
    if kind == "qwen32k":
        layer = kw.pop("layer", 0)
        kw.setdefault("batch", 2)
        kw.setdefault("length", 700)
        return make_qwen32k_layer(layer, seed, **kw)
    if kind == "hybrid":
        kw.setdefault("batch", 2)
        kw.setdefault("hist_len", 900)
        return make_hybrid(seed, **kw)
    raise ValueError(kind)


WORKLOADS: List[str] = ["tiny", "qwen4k", "qwen16k", "qwen32k", "hybrid"]
