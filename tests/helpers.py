"""Glue for the tests: feed one seeded synthetic problem to the CUDA library (through the
C ABI binding) and to the CPU oracle, and compare.  The oracle only ever sees
generator outputs; nothing it uses comes from the CUDA path."""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np

import synth
from oracle import attention, iskv, quant

# Tolerances (stated for the bf16 / int4 configurations: max-abs 2e-3 as the acceptance
# bar for bf16 inputs with fp32 accumulation, plus a relative bar of 1e-2 of the largest
# reference output and 1e-3 on the natural-log LSE, because the outputs of the qwen-shaped
# workloads are ~1e-4 and an absolute bar alone would accept zeros; 1e-5 for fp32).
TOL = {
    "f32": dict(abs=1e-5, rel=1e-5, lse=1e-5),
    "bf16": dict(abs=2e-3, rel=1e-2, lse=1e-3),
}


def fp16_operand_lse_bound(p: synth.Problem, q: np.ndarray) -> np.ndarray:
    """Worst-case |lse error| [B][Hq] of a decode whose tensor-core operands are the fp16
    roundings of q~ and of the dequantised int4 latents x^ (relative error <= 2^-11 each),
    with fp16 probabilities (<= 2^-11 in l) and fp32 accumulation:
      |d logit_t| <= s sum_i |(B_k,h q)_i| |x^_t,i| (2^-10 + (r + 2) 2^-24),
      |d lse|     <= max_t |d logit_t| + 2^-10.
    The derivation only bounds rounding; a wrong head, sign or index breaks it by orders
    of magnitude."""
    qv = stored_value(p, q)
    Bk = stored_value(p, p.B_k)
    d, G = p.head_dim, p.n_q_heads // p.n_kv_heads
    s = 1.0 / math.sqrt(d)
    eps = 2.0 ** -10 + (p.rank_k + 2) * 2.0 ** -24
    out = np.zeros((p.batch, p.n_q_heads))
    for b in range(p.batch):
        X = np.abs(oracle_latents(p, p.z_k[b]))
        for j in range(p.n_q_heads):
            h = j // G
            bq = np.abs(Bk[:, h * d:(h + 1) * d] @ qv[b, j])
            out[b, j] = s * np.max(X @ bq) * eps + 2.0 ** -10
    return out


def fp16_latent_rope_lse_bound(p: synth.Problem, q: np.ndarray) -> np.ndarray:
    """Worst-case |lse error| [B][Hq] of the keys-before-RoPE decode on tensor cores.  The
    keys are rebuilt from the fp16 roundings of the dequantised int4 latents x^ (error
    <= 2^-11 |x^| + 2^-25 each) and of B_k (bf16 -> fp16: exact above 2^-14, else <= 2^-25),
    accumulated in fp32 and rotated with the fp32 table; the rotated keys and the scaled
    query enter the score MMA as fp16 (each <= 2^-11 relative + 2^-25 absolute per element)
    with fp32 accumulation; the probabilities are fp16 as on the rank-space path.  With |.|
    the Euclidean norm (a rotation keeps it), b_i = |B_k,h[i, :]| and
    K_t = sum_i |x^_t,i| b_i (>= |k^_t|):
      E_t         = (3 2^-11 + (r + d + 8) 2^-24) K_t + 2^-25 sum_i b_i
                    + sqrt(d) 2^-25 (sum_i |x^_t,i| + 1),
      |d logit_t| <= s |q_j| E_t + sqrt(d) 2^-25 K_t,
      |d lse|     <= max_t |d logit_t| + 2^-10."""
    qv = stored_value(p, q)
    Bk = stored_value(p, p.B_k)
    d, G = p.head_dim, p.n_q_heads // p.n_kv_heads
    s = 1.0 / math.sqrt(d)
    rel = 3 * 2.0 ** -11 + (p.rank_k + d + 8) * 2.0 ** -24
    out = np.zeros((p.batch, p.n_q_heads))
    for b in range(p.batch):
        X = np.abs(oracle_latents(p, p.z_k[b]))
        sx = X.sum(axis=1)
        for h in range(p.n_kv_heads):
            bn = np.linalg.norm(Bk[:, h * d:(h + 1) * d], axis=1)
            K = X @ bn
            E = rel * K + 2.0 ** -25 * bn.sum() + math.sqrt(d) * 2.0 ** -25 * (sx + 1.0)
            for j in range(h * G, (h + 1) * G):
                out[b, j] = np.max(s * np.linalg.norm(qv[b, j]) * E + math.sqrt(d) * 2.0 ** -25 * K) + 2.0 ** -10
    return out


def decode_lse_bound(p: synth.Problem, q: np.ndarray) -> np.ndarray:
    """The LSE bar of a tensor-core decode over int4 latents: the rank-space bound or the
    keys-before-RoPE bound."""
    return fp16_latent_rope_lse_bound(p, q) if p.rope else fp16_operand_lse_bound(p, q)


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Oracle-side decoding of stored bf16 bit patterns (input format, not arithmetic)."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16)).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def stored_value(p: synth.Problem, x: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f64(x) if p.dtype == "bf16" else np.asarray(x, np.float64)


def oracle_latents(p: synth.Problem, z: np.ndarray) -> np.ndarray:
    """What the cache stores for fp32 latents z, by the oracle's own rules."""
    if p.quant_bits == 4:
        codes, scale, zero = quant.quantize_int4(z)
        return quant.dequantize_int4(codes, scale, zero, z.shape[-1])
    if p.dtype == "bf16":
        return quant.round_to_bf16(z)
    return np.asarray(z, np.float64)


def oracle_decode(p: synth.Problem, q: Optional[np.ndarray] = None, pairs=None,
                  rows: Optional[Sequence[int]] = None):
    """Oracle output for the problem as filled by `fill_cache`.  With `rows`, only those
    batch rows are materialised (the others are NaN)."""
    q = p.q if q is None else q
    qv = stored_value(p, q)
    Bsz = p.batch
    rows = list(range(Bsz)) if rows is None else list(rows)
    Zk = np.zeros((Bsz, p.hist_len, p.rank_k))
    Zv = np.zeros((Bsz, p.hist_len, p.rank_v))
    for b in rows:
        Zk[b] = oracle_latents(p, p.z_k[b])
        Zv[b] = oracle_latents(p, p.z_v[b])
    wk = stored_value(p, p.win_k) if p.win_k is not None else None
    wv = stored_value(p, p.win_v) if p.win_v is not None else None
    if pairs is None:
        pairs = [(b, j) for b in rows for j in range(p.n_q_heads)]
    return attention.decode(qv, Zk, Zv, stored_value(p, p.B_k), stored_value(p, p.B_v),
                            p.n_kv_heads, None, p.rope_theta if p.rope else None, wk, wv, pairs)


# ----------------------------------------------------------------------------
# device side
# ----------------------------------------------------------------------------


def to_dev(p: synth.Problem, x: np.ndarray):
    import torch
    if p.dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.cuda()


def desc_for(lr, p: synth.Problem, capacity: Optional[int] = None):
    return lr.make_desc(p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, p.rank_k, p.rank_v,
                        capacity or max(p.length + 8, p.window + 8), p.window, p.quant_bits,
                        lr.LR_BF16 if p.dtype == "bf16" else lr.LR_F32,
                        1 if p.rope else 0, p.rope_theta)


def fill_cache(lr, p: synth.Problem, capacity: Optional[int] = None, chunk: int = 0):
    """Create a cache for the problem and fill its history with the problem's latents
    (lr_kv_append_latent) and its window tokens (lr_kv_append)."""
    import torch
    c = lr.lr_cache_create(desc_for(lr, p, capacity), to_dev(p, p.A_k), to_dev(p, p.B_k),
                           to_dev(p, p.A_v), to_dev(p, p.B_v))
    n = p.hist_len
    step = chunk or n
    for s in range(0, n, max(step, 1)):
        e = min(n, s + step)
        zk = torch.from_numpy(np.ascontiguousarray(p.z_k[:, s:e])).cuda()
        zv = torch.from_numpy(np.ascontiguousarray(p.z_v[:, s:e])).cuda()
        lr.lr_kv_append_latent(c, zk, zv)
    for t in range(p.win_len):
        lr.lr_kv_append(c, to_dev(p, np.ascontiguousarray(p.win_k[:, t])),
                        to_dev(p, np.ascontiguousarray(p.win_v[:, t])))
    return c


def _value_layout_maps():
    """For the rank-major value blocks: word index within a rank row [32 ranks mod 8 ...] and
    nibble of token t, as the header defines them (XOR-rotated 16-byte columns; tokens
    2m, 2m+1 in nibbles m, m + 4)."""
    i = np.arange(256)[:, None]           # rank (only i // 2 % 4 matters)
    t = np.arange(128)[None, :]
    widx = (((t >> 5) ^ ((i >> 1) & 3)) << 2) + ((t & 31) >> 3)
    nib = ((t & 1) << 2) | ((t >> 1) & 3)
    return widx, nib[0]


def int4_token_major(lr, view, batch: int, which: str):
    """Copy a cache's int4 storage of K ("k") or V ("v") to the host and rearrange it from
    the blocked device layout to token-major ([B][tokens][G*4] code words, [B][tokens][G]
    {scale, zero} words), the layout of the oracle's packer.  Keys: [B][blocks][G][128][4]
    codes and [B][blocks][G][128] params.  Values: rank-major blocks [B][blocks][G*32][16]
    and per (block, group) 128 fp16 scales then 128 fp16 zeros."""
    nb = view.int4_blocks
    if which == "k":
        G = view.groups_k
        codes = lr.copy_view(view.codes_k, (batch, nb, G, 128, 4), "<i4")
        params = lr.copy_view(view.params_k, (batch, nb, G, 128), "<i4")
        c = codes.cpu().numpy().view(np.uint32).transpose(0, 1, 3, 2, 4).reshape(batch, nb * 128, G * 4)
        pr = params.cpu().numpy().view(np.uint32).transpose(0, 1, 3, 2).reshape(batch, nb * 128, G)
        return c, pr
    G = view.groups_v
    raw = lr.copy_view(view.codes_v, (batch, nb, G * 32, 16), "<i4").cpu().numpy().view(np.uint32)
    halves = lr.copy_view(view.params_v, (batch, nb, G, 128), "<i4").cpu().numpy().view(np.uint16)
    return value_blocks_to_token_major(raw, halves.reshape(batch, nb, G, 256))


def value_blocks_to_token_major(raw: np.ndarray, halves: np.ndarray):
    """raw [B][nb][G*32][16] u32 rank-major code rows, halves [B][nb][G][256] u16 (scales,
    then zeros) -> token-major code words [B][nb*128][G*4] and params [B][nb*128][G]."""
    batch, nb, R, _ = raw.shape
    G = R // 32
    widx, nib = _value_layout_maps()
    i_idx = np.arange(G * 32)[:, None]
    words = raw[:, :, i_idx, widx[(np.arange(G * 32) % 8)][:, :]]      # [B][nb][G*32][128]
    codes = (words >> (4 * nib[None, None, None, :]).astype(np.uint32)) & 15
    # token-major packing: element e of group g at word g*4 + e//8, nibble e%8
    codes = codes.transpose(0, 1, 3, 2).reshape(batch, nb * 128, G * 4, 8)
    c = np.zeros((batch, nb * 128, G * 4), np.uint32)
    for m in range(8):
        c |= codes[..., m].astype(np.uint32) << np.uint32(4 * m)
    sc = halves[..., :128].astype(np.uint32)
    zr = halves[..., 128:].astype(np.uint32)
    pr = (sc | (zr << 16)).transpose(0, 1, 3, 2).reshape(batch, nb * 128, G)
    return c, pr


def gpu_decode(lr, p: synth.Problem, cache, q: Optional[np.ndarray] = None, with_lse=True):
    import torch
    qd = to_dev(p, p.q if q is None else q)
    out = torch.empty_like(qd)
    lse = torch.empty((p.batch, p.n_q_heads), dtype=torch.float32, device="cuda") if with_lse else None
    lr.lr_attn_decode(cache, qd, out, lse)
    torch.cuda.synchronize()
    o = out.float().cpu().numpy().astype(np.float64)
    return o, (lse.cpu().numpy().astype(np.float64) if with_lse else None)


def compare(p: synth.Problem, got, ref, got_lse=None, ref_lse=None, pairs=None, tag="", lse_tol=None):
    """Assert the stated tolerances on the selected (b, j) outputs; return the errors.
    `lse_tol` ([B][Hq]) replaces the LSE bar where the decode's operands are rounded to
    fp16 (see fp16_operand_lse_bound)."""
    tol = TOL[p.dtype]
    lt = None
    if pairs is None:
        sel = np.isfinite(ref[..., 0])
        g, r = got[sel], ref[sel]
        gl = got_lse[sel] if got_lse is not None else None
        rl = ref_lse[sel] if ref_lse is not None else None
        lt = lse_tol[sel] if lse_tol is not None else None
    else:
        idx = tuple(np.array(pairs).T)
        g, r = got[idx], ref[idx]
        gl = got_lse[idx] if got_lse is not None else None
        rl = ref_lse[idx] if ref_lse is not None else None
        lt = lse_tol[idx] if lse_tol is not None else None
    assert np.all(np.isfinite(g)), f"{tag}: non-finite output"
    err = np.max(np.abs(g - r))
    scale = np.max(np.abs(r))
    assert err <= tol["abs"], f"{tag}: max abs err {err:.3e} > {tol['abs']}"
    assert err <= tol["rel"] * scale, f"{tag}: max abs err {err:.3e} > {tol['rel']} x {scale:.3e}"
    lerr = 0.0
    if gl is not None and rl is not None:
        lerr = np.max(np.abs(gl - rl))
        if lt is None:
            assert lerr <= tol["lse"], f"{tag}: lse err {lerr:.3e}"
        else:
            worst = np.max(np.abs(gl - rl) / np.maximum(lt, tol["lse"]))
            assert worst <= 1.0, f"{tag}: lse err {lerr:.3e} exceeds the fp16-operand bound (x{worst:.2f})"
    return err, err / max(scale, 1e-300), lerr


def sharp_factor(p: synth.Problem, target_std: float = 2.0) -> float:
    """Query multiplier that makes the logits' spread about `target_std` (natural-log
    units), so the softmax is far from uniform."""
    if p.hist_len < 2:
        return 1.0
    b = 0
    qv = stored_value(p, p.q)[b]
    Zk = oracle_latents(p, p.z_k[b][: min(256, p.hist_len)])
    Kh = Zk @ stored_value(p, p.B_k)[:, : p.head_dim]
    logits = Kh @ qv[0] / math.sqrt(p.head_dim)
    return float(target_std / max(np.std(logits), 1e-30))
