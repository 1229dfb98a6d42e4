"""Pins of the CPU oracle against facts fixed outside it: closed forms, invariants,
special cases, hand-derived values and brute force on tiny inputs."""
import json
import math
import os

import numpy as np
import pytest

import synth
from oracle import attention, iskv, quant, svd

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# quantiser and packing
# ----------------------------------------------------------------------------


def test_pack_every_nibble_in_every_position():
    for pos in range(8):
        for v in range(16):
            codes = np.zeros(8, np.uint8)
            codes[pos] = v
            w = quant.pack_nibbles(codes)
            assert w.shape == (1,)
            assert int(w[0]) == v << (4 * pos)
            assert np.array_equal(quant.unpack_nibbles(w), codes)


def test_pack_roundtrip_random():
    rng = np.random.default_rng(1)
    codes = rng.integers(0, 16, size=(5, 7, 64)).astype(np.uint8)
    assert np.array_equal(quant.unpack_nibbles(quant.pack_nibbles(codes)), codes)


def test_golden_ramp_hand_derived():
    g = json.load(open(os.path.join(GOLDEN, "quant_ramp.json")))
    x = np.asarray(g["x"], np.float32)[None]
    codes, scale, zero = quant.quantize_int4(x)
    assert float(scale[0, 0]) == g["scale"]
    assert float(zero[0, 0]) == g["zero"]
    assert codes[0].tolist() == g["codes"]
    assert quant.pack_nibbles(codes)[0].tolist() == g["words"]
    deq = quant.dequantize_int4(codes, scale, zero, 32)[0]
    assert np.array_equal(deq, np.floor(np.arange(32) / 2) * g["scale"])


def test_constant_group_codes_zero():
    x = np.full((3, 32), 3.25, np.float32)
    codes, scale, zero = quant.quantize_int4(x)
    assert np.all(codes == 0) and np.all(scale == 0) and np.all(zero == np.float16(3.25))
    assert np.all(quant.dequantize_int4(codes, scale, zero, 32) == 3.25)


def test_integer_group_exact_min_max():
    # values 0..15 with scale exactly 1: codes equal the values, min -> 0, max -> 15
    rng = np.random.default_rng(2)
    v = np.concatenate([[0, 15], rng.integers(0, 16, 30)]).astype(np.float32)
    rng.shuffle(v)
    codes, scale, zero = quant.quantize_int4(v[None] + 100.0)
    assert float(scale[0, 0]) == 1.0 and float(zero[0, 0]) == 100.0
    assert np.array_equal(codes[0].astype(np.float32), v)


def test_ties_round_to_even():
    # zero 0, scale 1 (min 0, max 15); x = k + 0.5 must go to the even neighbour
    x = np.zeros(32, np.float32)
    x[0], x[1] = 0.0, 15.0
    halves = np.arange(14) + 0.5
    x[2:16] = halves
    codes, scale, zero = quant.quantize_int4(x[None])
    assert float(scale[0, 0]) == 1.0 and float(zero[0, 0]) == 0.0
    expect = [int(2 * round(h / 2)) for h in halves]          # nearest even integer
    assert codes[0, 2:16].tolist() == expect
    assert codes[0, 2] == 0 and codes[0, 3] == 2 and codes[0, 4] == 2


def test_signed_zero_and_negative_range():
    x = np.zeros(32, np.float32)
    x[::2] = -0.0
    codes, scale, zero = quant.quantize_int4(x[None])
    assert np.all(codes == 0) and float(scale[0, 0]) == 0.0
    assert zero.view(np.uint16)[0, 0] == 0          # zero point stored as +0, not -0
    _, _, z2 = quant.quantize_int4(np.full((1, 32), -0.0, np.float32))
    assert z2.view(np.uint16)[0, 0] == 0
    y = np.linspace(-7.5, 0.0, 32).astype(np.float32)   # min -7.5 -> code 0, max 0 -> 15
    codes, scale, zero = quant.quantize_int4(y[None])
    assert codes[0, 0] == 0 and codes[0, -1] == 15 and float(zero[0, 0]) == -7.5
    assert float(scale[0, 0]) == 0.5


def test_partial_last_group_uses_only_real_elements():
    r = 48                       # a multiple of 16 with a half group at the end
    x = np.zeros(r, np.float32)
    x[:32] = np.linspace(-1000, 1000, 32)
    x[32:] = 100 + np.arange(16)                    # second group: 100..115
    codes, scale, zero = quant.quantize_int4(x[None])
    assert codes.shape == (1, 64) and scale.shape == (1, 2)
    assert float(zero[0, 1]) == 100.0 and float(scale[0, 1]) == 1.0
    assert codes[0, 32:48].tolist() == list(range(16))
    assert np.all(codes[0, 48:] == 0)
    words = quant.pack_nibbles(codes)
    assert words.shape == (1, 8) and words[0, 6] == 0 and words[0, 7] == 0


def test_group_to_word_mapping():
    # three groups; group g holds codes (e + g) % 16 -> word 4g + e // 8, nibble e % 8
    r = 96
    codes = np.array([[(e + g) % 16 for g in range(3) for e in range(32)]], np.uint8)
    words = quant.pack_nibbles(codes)
    for g in range(3):
        for e in range(32):
            w = int(words[0, 4 * g + e // 8])
            assert (w >> (4 * (e % 8))) & 0xF == (e + g) % 16
    assert r == codes.shape[1]


def test_dequant_error_bound():
    rng = np.random.default_rng(3)
    z = (rng.standard_normal((64, 352)) * synth.spectrum(352, 0.7)).astype(np.float32)
    codes, scale, zero = quant.quantize_int4(z)
    xh = quant.dequantize_int4(codes, scale, zero, 352)
    gi = np.arange(352) // 32
    s = scale.astype(np.float64)[:, gi]
    zz = zero.astype(np.float64)[:, gi]
    zr = z.astype(np.float64).reshape(64, 11, 32)
    mn = np.repeat(zr.min(-1), 32, axis=1)
    mx = np.repeat(zr.max(-1), 32, axis=1)
    exact_scale = (mx - mn) / 15
    bound = s / 2 + np.abs(mn - zz) + 15 * np.abs(s - exact_scale) + 1e-6 * (np.abs(mx) + np.abs(mn))
    err = np.abs(z - xh)
    assert np.all(err <= bound)
    assert np.all(codes <= 15)


# ----------------------------------------------------------------------------
# bf16 storage rounding: two independent implementations must agree
# ----------------------------------------------------------------------------


def test_bf16_rounding_hand_cases():
    assert quant.round_to_bf16_scalar(1 + 2 ** -8) == 1.0                 # tie -> even (down)
    assert quant.round_to_bf16_scalar(1 + 3 * 2 ** -8) == 1 + 2 ** -6     # tie -> even (up)
    assert quant.round_to_bf16_scalar(1 + 2 ** -8 + 2 ** -20) == 1 + 2 ** -7
    assert quant.round_to_bf16_scalar(-3.0) == -3.0


def test_bf16_rounding_matches_generator():
    rng = np.random.default_rng(4)
    x = rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))
    base = synth.bf16_to_f64(synth.bf16_bits(x))
    # exact ties: bf16 value plus half an ulp
    ties = base + np.ldexp(1.0, np.frexp(base)[1] - 9)
    for arr in (x, ties):
        a = quant.round_to_bf16(arr)
        b = synth.bf16_to_f64(synth.bf16_bits(arr))
        assert np.array_equal(a, b)
        sc = np.array([quant.round_to_bf16_scalar(v) for v in arr[:500]])
        assert np.array_equal(sc, a[:500])


# ----------------------------------------------------------------------------
# attention definition
# ----------------------------------------------------------------------------


def _brute_latent_decode(q, Zk, Zv, Bk, Bv, Hkv, scale):
    """Pure-Python loops over the latent-space form of the same attention:
    q~ = B_k,h q ; s_t = q~ . z_t ; o~ = sum_t w_t z_v,t ; o = o~ B_v,h."""
    Bsz, Hq, d = q.shape
    T = Zk.shape[1]
    out = np.zeros((Bsz, Hq, d))
    lse = np.zeros((Bsz, Hq))
    for b in range(Bsz):
        for j in range(Hq):
            h = j // (Hq // Hkv)
            qt = [sum(Bk[i][h * d + c] * q[b][j][c] for c in range(d)) for i in range(Bk.shape[0])]
            logits = [scale * sum(qt[i] * Zk[b][t][i] for i in range(len(qt))) for t in range(T)]
            m = max(logits)
            e = [math.exp(x - m) for x in logits]
            l = sum(e)
            ot = [sum(e[t] / l * Zv[b][t][i] for t in range(T)) for i in range(Bv.shape[0])]
            for c in range(d):
                out[b, j, c] = sum(ot[i] * Bv[i][h * d + c] for i in range(len(ot)))
            lse[b, j] = m + math.log(l)
    return out, lse


def test_decode_matches_brute_force_latent_form():
    rng = np.random.default_rng(5)
    Bsz, Hq, Hkv, d, rk, rv, T = 2, 4, 2, 4, 3, 5, 3
    q = rng.standard_normal((Bsz, Hq, d))
    Zk = rng.standard_normal((Bsz, T, rk))
    Zv = rng.standard_normal((Bsz, T, rv))
    Bk = rng.standard_normal((rk, Hkv * d))
    Bv = rng.standard_normal((rv, Hkv * d))
    o1, l1 = attention.decode(q, Zk, Zv, Bk, Bv, Hkv, 0.7)
    o2, l2 = _brute_latent_decode(q, Zk, Zv, Bk, Bv, Hkv, 0.7)
    assert np.max(np.abs(o1 - o2)) < 1e-12 and np.max(np.abs(l1 - l2)) < 1e-12


def test_single_token_returns_value_exactly():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((1, 2, 8))
    Zk = rng.standard_normal((1, 1, 4))
    Zv = rng.standard_normal((1, 1, 4))
    Bk = rng.standard_normal((4, 8))
    Bv = rng.standard_normal((4, 8))
    o, lse = attention.decode(q, Zk, Zv, Bk, Bv, 1)
    v = Zv[0, 0] @ Bv
    assert np.allclose(o[0, 0], v, rtol=0, atol=1e-14) and np.allclose(o[0, 1], v, atol=1e-14)
    logit = (Zk[0, 0] @ Bk) @ q[0, 0] / math.sqrt(8)
    assert abs(lse[0, 0] - logit) < 1e-12


def test_two_tokens_sigmoid_closed_form():
    k1, k2 = np.array([1.0, 0.0]), np.array([0.0, 2.0])
    v1, v2 = np.array([3.0, -1.0]), np.array([0.5, 4.0])
    q = np.array([0.3, -0.8])
    o, lse, w = attention.softmax_attention(q, np.stack([k1, k2]), np.stack([v1, v2]), 1.0)
    l1, l2 = q @ k1, q @ k2
    w1 = 1.0 / (1.0 + math.exp(l2 - l1))
    assert abs(w[0] - w1) < 1e-15 and abs(w.sum() - 1) < 1e-15
    assert np.allclose(o, w1 * v1 + (1 - w1) * v2, atol=1e-15)
    assert abs(lse - math.log(math.exp(l1) + math.exp(l2))) < 1e-14


def test_equal_keys_average_values_and_weights_sum_to_one():
    rng = np.random.default_rng(7)
    K = np.tile(rng.standard_normal(6), (50, 1))
    V = rng.standard_normal((50, 6))
    o, lse, w = attention.softmax_attention(rng.standard_normal(6), K, V, 0.5)
    assert np.allclose(o, V.mean(0), atol=1e-14)
    K2 = rng.standard_normal((300, 6)) * 5
    _, _, w2 = attention.softmax_attention(rng.standard_normal(6), K2, V.repeat(6, 0), 1.0)
    assert abs(w2.sum() - 1) < 1e-12


def test_full_rank_identity_bases_equal_dense_attention():
    # r = D with A = B = I: latents are the keys themselves (config-1 shape at full rank)
    rng = np.random.default_rng(8)
    T, d = 256, 64
    K = rng.standard_normal((1, T, d))
    V = rng.standard_normal((1, T, d))
    q = rng.standard_normal((1, 2, d))
    I = np.eye(d)
    o, lse = attention.decode(q, K, V, I, I, 1)
    for j in range(2):
        logits = [sum(q[0, j, c] * K[0, t, c] for c in range(d)) / 8.0 for t in range(T)]
        m = max(logits)
        e = [math.exp(x - m) for x in logits]
        l = sum(e)
        ref = [sum(e[t] * V[0, t, c] for t in range(T)) / l for c in range(d)]
        assert np.max(np.abs(o[0, j] - np.array(ref))) < 1e-12


def test_gqa_head_mapping_contiguous_groups():
    rng = np.random.default_rng(9)
    Bsz, Hq, Hkv, d, r, T = 1, 6, 3, 4, 5, 7
    q = rng.standard_normal((Bsz, Hq, d))
    q[0, 1] = q[0, 0]                                # heads 0, 1 share KV head 0
    Zk, Zv = rng.standard_normal((Bsz, T, r)), rng.standard_normal((Bsz, T, r))
    Bk, Bv = rng.standard_normal((r, Hkv * d)), rng.standard_normal((r, Hkv * d))
    o, _ = attention.decode(q, Zk, Zv, Bk, Bv, Hkv)
    assert np.array_equal(o[0, 0], o[0, 1])
    Bk2 = Bk.copy()
    Bk2[:, 2 * d:3 * d] += 1.0                       # perturb KV head 2 only
    o2, _ = attention.decode(q, Zk, Zv, Bk2, Bv, Hkv)
    assert np.array_equal(o2[0, :4], o[0, :4])        # query heads 0..3 -> KV heads 0, 1
    assert not np.allclose(o2[0, 4:], o[0, 4:])


def test_window_only_equals_dense_attention():
    rng = np.random.default_rng(10)
    Bsz, Hq, Hkv, d, W = 1, 2, 1, 8, 5
    wk, wv = rng.standard_normal((Bsz, W, d)), rng.standard_normal((Bsz, W, d))
    q = rng.standard_normal((Bsz, Hq, d))
    o, _ = attention.decode(q, np.zeros((1, 0, 3)), np.zeros((1, 0, 3)), np.zeros((3, d)),
                            np.zeros((3, d)), Hkv, None, None, wk, wv)
    for j in range(Hq):
        ref, _, _ = attention.softmax_attention(q[0, j], wk[0], wv[0], 1 / math.sqrt(d))
        lg = [float(q[0, j] @ wk[0, t]) / math.sqrt(d) for t in range(W)]
        e = [math.exp(x - max(lg)) for x in lg]
        bf = sum(e[t] * wv[0, t] for t in range(W)) / sum(e)
        assert np.allclose(o[0, j], bf, atol=1e-14) and np.allclose(ref, bf, atol=1e-14)


# ----------------------------------------------------------------------------
# RoPE
# ----------------------------------------------------------------------------


def test_rope_closed_forms():
    x = np.array([[0.6, -1.3]])
    for t in (0, 1, 5, 1000):
        y = attention.rope_rotate_half(x, np.array([t]), 1e6)
        c, s = math.cos(t), math.sin(t)                 # d = 2: omega_0 = 1
        assert np.allclose(y[0], [0.6 * c + 1.3 * s, -1.3 * c + 0.6 * s], atol=1e-15)
    x4 = np.array([[1.0, 2.0, 3.0, 4.0]])
    th = 100.0
    y = attention.rope_rotate_half(x4, np.array([3]), th)
    a0, a1 = 3.0, 3.0 * th ** -0.5                      # omega = (1, theta^(-1/2))
    exp = [1 * math.cos(a0) - 3 * math.sin(a0), 2 * math.cos(a1) - 4 * math.sin(a1),
           3 * math.cos(a0) + 1 * math.sin(a0), 4 * math.cos(a1) + 2 * math.sin(a1)]
    assert np.allclose(y[0], exp, atol=1e-14)


def test_rope_invariants():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((40, 128))
    pos = rng.integers(0, 40000, 40)
    assert np.array_equal(attention.rope_rotate_half(x, np.zeros(40), 1e6), x)
    y = attention.rope_rotate_half(x, pos, 1e6)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    q, k = rng.standard_normal((1, 128)), rng.standard_normal((1, 128))
    s1 = attention.rope_rotate_half(q, [700], 1e6) @ attention.rope_rotate_half(k, [200], 1e6).T
    s2 = attention.rope_rotate_half(q, [10500], 1e6) @ attention.rope_rotate_half(k, [10000], 1e6).T
    assert abs(s1[0, 0] - s2[0, 0]) < 1e-10


def test_decode_with_rope_matches_rotated_dense():
    rng = np.random.default_rng(12)
    T, d, r = 9, 8, 8
    Zk, Zv = rng.standard_normal((1, T, r)), rng.standard_normal((1, T, r))
    Bk, Bv = np.eye(r), np.eye(r)
    q = rng.standard_normal((1, 1, d))
    o, _ = attention.decode(q, Zk, Zv, Bk, Bv, 1, None, 1e4)
    Kr = attention.rope_rotate_half(Zk[0], np.arange(T), 1e4)
    ref, _, _ = attention.softmax_attention(q[0, 0], Kr, Zv[0], 1 / math.sqrt(d))
    assert np.allclose(o[0, 0], ref, atol=1e-14)
    # positions matter: the unrotated cache gives a different answer
    o0, _ = attention.decode(q, Zk, Zv, Bk, Bv, 1)
    assert not np.allclose(o0, o)


# ----------------------------------------------------------------------------
# truncated SVD: Eckart-Young closed form on matrices of known spectrum
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("r", [1, 8, 32, 63])
def test_eckart_young_closed_form(r):
    rng = np.random.default_rng(13)
    T, D = 200, 64
    sig = synth.spectrum(D, 0.8) * 3.0
    U = synth.haar_orthonormal(rng, D, T).T        # [T][D] orthonormal columns
    W = synth.haar_orthogonal(rng, D)
    X = (U * sig[None, :]) @ W
    A, B, s = svd.truncated_basis(X, r)
    fro, spec = svd.lowrank_residual(X, A, B)
    assert abs(fro - np.sqrt(np.sum(sig[r:] ** 2))) <= 1e-10 * np.linalg.norm(sig)
    assert abs(spec - sig[r]) <= 1e-10 * sig[0]
    assert np.allclose(s, sig, rtol=1e-10)
    f2, s2 = svd.eckart_young(sig, r)
    assert abs(f2 - fro) < 1e-10 and abs(s2 - spec) < 1e-10


def test_tiny_workload_bases_are_optimal():
    p = synth.make_tiny()
    K = p.extra["K"][0].astype(np.float64)
    _, _, s = svd.truncated_basis(K, p.rank_k)
    fro, _ = svd.lowrank_residual(K, p.A_k.astype(np.float64), p.B_k.astype(np.float64))
    best, _ = svd.eckart_young(s, p.rank_k)
    assert abs(fro - best) <= 1e-5 * np.linalg.norm(s)


# ----------------------------------------------------------------------------
# windowed cache (iS-KV reading)
# ----------------------------------------------------------------------------


def _hybrid_small(W=4, r=6, Hkv=2, d=4, Bsz=2):
    rng = np.random.default_rng(14)
    D = Hkv * d
    Bk = synth.haar_orthonormal(rng, r, D) / math.sqrt(r)
    Bv = synth.haar_orthonormal(rng, r, D) / math.sqrt(r)
    return rng, Bk, Bv, r * Bk.T, r * Bv.T, D


def test_fold_is_exact_for_tokens_in_the_subspace():
    rng, Bk, Bv, Ak, Av, D = _hybrid_small()
    sim = iskv.WindowedCacheSim(Ak, Bk, Av, Bv, 2, 4, "f32")
    toks = []
    for t in range(11):
        g = rng.standard_normal((2, 6))
        k, v = g @ Bk, (g * 0.5) @ Bv
        toks.append((k, v))
        sim.append(k, v)
    assert sim.length == 11 and sim.hist_k.shape[1] == 7 and len(sim.win_k) == 4
    for t in range(7):                       # folded tokens reconstruct to themselves
        assert np.allclose(sim.hist_k[:, t] @ Bk, toks[t][0], atol=1e-6)
        assert np.allclose(sim.hist_v[:, t] @ Bv, toks[t][1], atol=1e-6)
    for i, t in enumerate(range(7, 11)):     # window keeps the last four exactly (fp32)
        assert np.allclose(sim.win_k[i], toks[t][0], atol=1e-6)


def test_sync_invariance_identity_and_drift():
    rng, Bk, Bv, Ak, Av, D = _hybrid_small()
    sim = iskv.WindowedCacheSim(Ak, Bk, Av, Bv, 2, 4, "f32")
    sim.store = lambda x: np.asarray(x, np.float64)          # exact storage for the invariant
    for t in range(12):
        g = rng.standard_normal((2, 6))
        sim.append(g @ Bk + 0.01 * rng.standard_normal((2, D)), g @ Bv)
    q = rng.standard_normal((2, 4, 4)) * 3
    before, lse0 = sim.decode(q)
    Rk, Rv = synth.haar_orthogonal(rng, 6), synth.haar_orthogonal(rng, 6)
    hk = sim.hist_k.copy()
    sim.sync(np.eye(6), np.eye(6))
    assert np.array_equal(sim.hist_k, hk)                    # R = I leaves latents unchanged
    drift = iskv.WindowedCacheSim(Ak, Rk.T @ Bk, Av, Rv.T @ Bv, 2, 4, "f32")
    drift.store = sim.store
    drift.hist_k, drift.hist_v = sim.hist_k.copy(), sim.hist_v.copy()
    drift.win_k, drift.win_v = list(sim.win_k), list(sim.win_v)
    moved, _ = drift.decode(q)                               # new basis, stale coordinates
    assert np.max(np.abs(moved - before)) > 1e-3
    sim.sync(Rk, Rv, Rk.T @ Bk, Rv.T @ Bv, Ak @ Rk, Av @ Rv)
    after, lse1 = sim.decode(q)
    assert np.max(np.abs(after - before)) < 1e-12 and np.max(np.abs(lse1 - lse0)) < 1e-12


def test_window_larger_than_length_is_dense_attention():
    rng, Bk, Bv, Ak, Av, D = _hybrid_small()
    sim = iskv.WindowedCacheSim(Ak, Bk, Av, Bv, 2, 16, "f32")
    ks, vs = [], []
    for t in range(5):
        k, v = rng.standard_normal((2, D)), rng.standard_normal((2, D))
        sim.append(k, v)
        ks.append(sim.win_k[-1])
        vs.append(sim.win_v[-1])
    q = rng.standard_normal((2, 4, 4))
    o, _ = sim.decode(q)
    K, V = np.stack(ks, 1), np.stack(vs, 1)
    for b in range(2):
        for j in range(4):
            h = j // 2
            ref, _, _ = attention.softmax_attention(q[b, j], K[b][:, h * 4:(h + 1) * 4],
                                                    V[b][:, h * 4:(h + 1) * 4], 0.5)
            assert np.allclose(o[b, j], ref, atol=1e-14)


def test_latent_identity():
    rng = np.random.default_rng(15)
    Bh = rng.standard_normal((32, 16))
    q, z = rng.standard_normal(16), rng.standard_normal(32)
    lhs = q @ (z @ Bh)
    rhs = (Bh @ q) @ z
    assert abs(lhs - rhs) <= 1e-12 * (np.abs(Bh).sum() * np.abs(q).max() * np.abs(z).max())
