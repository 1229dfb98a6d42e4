"""CPU checks of the rounding bounds that serve as LSE bars for the int4 tensor-core decode
paths (`helpers.fp16_operand_lse_bound`, `helpers.fp16_latent_rope_lse_bound`).

Each test runs an independent NumPy emulation of one kernel's arithmetic: fp16 roundings of
its tensor-core operands, fp32 accumulation, fp32 rotation factors from fp64 angles, fp32
exponentials rounded to fp16 probabilities, an fp32 normaliser.  The emulated LSE must lie
within the bound of the fp64 oracle's LSE for every (sequence, head), and an emulation with a
planted mistake (wrong rotation sign, wrong KV head) must land far outside it, so the bound
is tight enough to catch the mistakes it is meant to catch."""
import math

import numpy as np
import pytest

import synth
from tests import helpers as H

LN2 = math.log(2.0)
LOG2E = 1.0 / LN2


def _fp16(x) -> np.ndarray:
    """Round to fp16 (nearest even), held in fp32."""
    return np.asarray(x, np.float64).astype(np.float16).astype(np.float32)


def _lse_from_log2_logits(s2: np.ndarray) -> float:
    """LSE (natural log) of one row of base-2 logits the way the kernels finish it: fp32
    exponentials relative to the row max, rounded to fp16, summed in fp32."""
    s2 = np.asarray(s2, np.float32)
    m = np.float32(s2.max())
    p = _fp16(np.exp2(s2 - m))
    l = np.float32(p.sum(dtype=np.float32))
    return (float(m) + math.log2(float(l))) * LN2


def _scaled_queries(p: synth.Problem, q: np.ndarray) -> np.ndarray:
    """fp32(q * s log2(e)), as the query kernels store it."""
    return H.stored_value(p, q).astype(np.float32) * np.float32(LOG2E / math.sqrt(p.head_dim))


def _emulate_rank_space(p: synth.Problem, q: np.ndarray, head_shift: int = 0) -> np.ndarray:
    """int4 latents, keys after RoPE: S = fp16(x^) . fp16(q~) with q~ = B_k,h q s log2(e) in fp32."""
    d, Hq, Hkv = p.head_dim, p.n_q_heads, p.n_kv_heads
    G = Hq // Hkv
    Bk = H.stored_value(p, p.B_k).astype(np.float32)
    qs = _scaled_queries(p, q)
    lse = np.zeros((p.batch, Hq))
    for b in range(p.batch):
        x16 = _fp16(H.oracle_latents(p, p.z_k[b]))
        for j in range(Hq):
            h = (j // G + head_shift) % Hkv
            qt16 = _fp16(Bk[:, h * d:(h + 1) * d] @ qs[b, j])
            lse[b, j] = _lse_from_log2_logits(x16 @ qt16)
    return lse


def _emulate_rope(p: synth.Problem, q: np.ndarray, sin_sign: float = 1.0, head_shift: int = 0) -> np.ndarray:
    """int4 latents, keys before RoPE: K^ = fp16(x^) fp16(B_k) in fp32, rotate-half with an
    fp32 cos / sin table, the rotated keys and the scaled query rounded to fp16, dots
    accumulated in fp32."""
    d, Hq, Hkv = p.head_dim, p.n_q_heads, p.n_kv_heads
    G, half = Hq // Hkv, p.head_dim // 2
    B16 = _fp16(H.stored_value(p, p.B_k))
    qs = _scaled_queries(p, q)
    T = p.hist_len
    omega = p.rope_theta ** (-2.0 * np.arange(half) / d)
    ang = np.arange(T)[:, None] * omega[None, :]
    cos = np.cos(ang).astype(np.float32)
    sin = (sin_sign * np.sin(ang)).astype(np.float32)
    lse = np.zeros((p.batch, Hq))
    for b in range(p.batch):
        K = _fp16(H.oracle_latents(p, p.z_k[b])) @ B16
        for j in range(Hq):
            h = (j // G + head_shift) % Hkv
            k1, k2 = K[:, h * d:h * d + half], K[:, h * d + half:(h + 1) * d]
            kr = _fp16(np.concatenate([k1 * cos - k2 * sin, k2 * cos + k1 * sin], axis=1))
            lse[b, j] = _lse_from_log2_logits(kr @ _fp16(qs[b, j]))
    return lse


def _ratio(emul, ref, bound):
    return np.abs(emul - ref) / bound


def _sharp(p):
    return p.store(H.stored_value(p, p.q) * H.sharp_factor(p))


@pytest.fixture(scope="module")
def rank_space():
    return synth.small_variant("qwen16k", length=600)


@pytest.fixture(scope="module")
def rope():
    return synth.small_variant("qwen32k", layer=0, length=300)


@pytest.mark.parametrize("sharp", [False, True])
def test_rank_space_bound_holds_for_emulated_kernel(rank_space, sharp):
    p = rank_space
    q = _sharp(p) if sharp else p.q
    _, ref = H.oracle_decode(p, q)
    r = _ratio(_emulate_rank_space(p, q), ref, H.fp16_operand_lse_bound(p, q))
    assert np.max(r) <= 1.0, np.max(r)


@pytest.mark.parametrize("sharp", [False, True])
def test_rope_bound_holds_for_emulated_kernel(rope, sharp):
    p = rope
    q = _sharp(p) if sharp else p.q
    _, ref = H.oracle_decode(p, q)
    r = _ratio(_emulate_rope(p, q), ref, H.fp16_latent_rope_lse_bound(p, q))
    assert np.max(r) <= 1.0, np.max(r)


def test_rank_space_bound_catches_a_wrong_head(rank_space):
    p = rank_space
    q = _sharp(p)
    _, ref = H.oracle_decode(p, q)
    r = _ratio(_emulate_rank_space(p, q, head_shift=1), ref, H.fp16_operand_lse_bound(p, q))
    assert np.max(r) > 10.0, np.max(r)


@pytest.mark.parametrize("mistake", [dict(sin_sign=-1.0), dict(head_shift=1)])
def test_rope_bound_catches_planted_mistakes(rope, mistake):
    p = rope
    q = _sharp(p)
    _, ref = H.oracle_decode(p, q)
    r = _ratio(_emulate_rope(p, q, **mistake), ref, H.fp16_latent_rope_lse_bound(p, q))
    assert np.max(r) > 10.0, np.max(r)
