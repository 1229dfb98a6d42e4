"""Latent quantisation and storage rounding (oracle side).

TraceKV abstract: low-rank latents "can be combined with quantization"; the
digest's Synopsis gives the operating point (70% rank ratio with 4-bit
quantization).  The pages define no quantiser, so this module follows the
plainest reading of a 4-bit asymmetric group quantiser:

  for each group of (up to) 32 consecutive latent coordinates of one token,
    mn, mx  = min, max over the group's real elements (fp32 values)
    zero    = fp16(mn)                       (round to nearest even; -0 stored as +0)
    scale   = fp16((mx - mn) / 15)           (fp32 subtract, fp32 divide, then fp16)
    code    = 0                               if scale == 0
            = clamp(rint((x - zero) / scale), 0, 15)   otherwise,
              with x - zero and the division done in IEEE fp32 and rint ties to even
  dequantised value  x^ = code * scale + zero  (exact in fp64)

Packing: group g of a token occupies 4 uint32 words; element e of the group is
stored in word 4g + e // 8 at bits 4 (e mod 8) .. 4 (e mod 8) + 3 (low nibble
first).  A final partial group keeps its unused nibbles at zero.
"""
from __future__ import annotations

import math

import numpy as np

GROUP = 32
WORDS_PER_GROUP = GROUP // 8


def n_groups(r: int, group: int = GROUP) -> int:
    return (r + group - 1) // group


def quantize_int4(z: np.ndarray, group: int = GROUP):
    """Quantise fp32 latents [..., r] -> (codes uint8 [..., G*group], scale f16 [..., G],
    zero f16 [..., G]).  Codes of the padding positions are 0."""
    z = np.asarray(z, dtype=np.float32)
    r = z.shape[-1]
    G = n_groups(r, group)
    lead = z.shape[:-1]
    codes = np.zeros(lead + (G * group,), dtype=np.uint8)
    scale = np.zeros(lead + (G,), dtype=np.float16)
    zero = np.zeros(lead + (G,), dtype=np.float16)
    fifteen = np.float32(15.0)
    for g in range(G):
        lo, hi = g * group, min(r, (g + 1) * group)
        seg = z[..., lo:hi]
        mn = seg.min(axis=-1)
        mx = seg.max(axis=-1)
        zg = mn.astype(np.float16)
        zg = np.where(zg == 0, np.float16(0.0), zg)      # a -0 zero point is stored as +0
        sg = ((mx - mn) / fifteen).astype(np.float16)   # fp32 ops, then fp16 rounding
        zero[..., g] = zg
        scale[..., g] = sg
        zf = zg.astype(np.float32)[..., None]
        sf = sg.astype(np.float32)[..., None]
        with np.errstate(divide="ignore", invalid="ignore"):
            t = (seg - zf) / sf                         # fp32 subtract and divide
            c = np.rint(t)                              # ties to even
        c = np.clip(c, 0, 15)
        c = np.where(sf == 0, 0, c)
        codes[..., lo:hi] = c.astype(np.uint8)
    return codes, scale, zero


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """uint8 codes [..., n] (n a multiple of 8, values < 16) -> uint32 words [..., n/8]."""
    codes = np.asarray(codes, dtype=np.uint32)
    n = codes.shape[-1]
    assert n % 8 == 0
    c = codes.reshape(codes.shape[:-1] + (n // 8, 8))
    words = np.zeros(c.shape[:-1], dtype=np.uint32)
    for e in range(8):
        words |= (c[..., e] & 0xF) << np.uint32(4 * e)
    return words


def unpack_nibbles(words: np.ndarray) -> np.ndarray:
    """uint32 words [..., w] -> uint8 codes [..., 8w]."""
    words = np.asarray(words, dtype=np.uint32)
    out = np.zeros(words.shape + (8,), dtype=np.uint8)
    for e in range(8):
        out[..., e] = (words >> np.uint32(4 * e)) & 0xF
    return out.reshape(words.shape[:-1] + (words.shape[-1] * 8,))


def dequantize_int4(codes: np.ndarray, scale: np.ndarray, zero: np.ndarray, r: int,
                    group: int = GROUP) -> np.ndarray:
    """Exact fp64 dequantisation x^ = code * scale + zero for the first r coordinates."""
    c = np.asarray(codes, dtype=np.float64)[..., :r]
    gi = np.arange(r) // group
    s = np.asarray(scale, dtype=np.float64)[..., gi]
    zz = np.asarray(zero, dtype=np.float64)[..., gi]
    return c * s + zz


def quantize_and_pack(z: np.ndarray, group: int = GROUP):
    """-> (words uint32 [..., G*4], scale f16 [..., G], zero f16 [..., G])."""
    codes, scale, zero = quantize_int4(z, group)
    return pack_nibbles(codes), scale, zero


# ----------------------------------------------------------------------------
# bf16 storage rounding, written independently of the input generator: round the
# significand to 8 bits with ties to even, using frexp/ldexp on fp64 values.
# ----------------------------------------------------------------------------


def _round_sig_bits(x: float, bits: int) -> float:
    if x == 0.0 or not math.isfinite(x):
        return x
    m, e = math.frexp(x)                 # x = m * 2^e, 0.5 <= |m| < 1
    scaled = m * (1 << bits)             # exact
    rounded = round(scaled)              # Python round(): ties to even
    return math.ldexp(rounded, e - bits)


def round_to_bf16(x) -> np.ndarray:
    """fp64 values -> fp64 value of the nearest bf16 (ties to even), for normal-range
    inputs.  The value is first rounded to fp32, as a store of an fp32 result would."""
    a = np.asarray(x, dtype=np.float64)
    a32 = a.astype(np.float32).astype(np.float64)
    m, e = np.frexp(a32)
    scaled = m * 256.0                   # 8 significant bits
    rounded = np.rint(scaled)            # ties to even
    return np.ldexp(rounded, e - 8)


def round_to_bf16_scalar(x: float) -> float:
    """Scalar reference of round_to_bf16 (pure Python), used by the pins."""
    return _round_sig_bits(float(np.float32(x)), 8)
