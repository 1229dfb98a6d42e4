"""The prefill epilogue's int4 code without a division per element: y = x * RN(1/s) decides
rint(RN(x / s)) unless y lies within 1e-5 of a half-integer, where the division decides.
Emulated here in IEEE fp32 (NumPy float32 arithmetic rounds to nearest even, as the GPU's
fp32 multiply, reciprocal and division do) against the division path the append quantiser
takes, on random groups and on quotients placed at and next to every half-integer."""
import numpy as np


def by_division(x, s):
    q = np.rint(np.divide(x, s, dtype=np.float32))
    return np.clip(q, 0, 15).astype(np.int64)


def by_reciprocal(x, s):
    rs = np.divide(np.float32(1.0), s, dtype=np.float32)
    y = np.multiply(x, rs, dtype=np.float32)
    off = np.abs(y - np.floor(y) - np.float32(0.5))
    q = np.where(off < np.float32(1e-5), np.rint(np.divide(x, s, dtype=np.float32)), np.rint(y))
    return np.clip(q, 0, 15).astype(np.int64)


def test_random_groups():
    rng = np.random.default_rng(0)
    for _ in range(200):
        z = (rng.standard_normal(32) * rng.uniform(1e-3, 10)).astype(np.float32)
        zf = np.float32(np.float16(z.min()))
        s = np.float32(np.float16(np.float32(z.max() - z.min()) / np.float32(15)))
        if s == 0:
            continue
        x = np.subtract(z, zf, dtype=np.float32)
        assert np.array_equal(by_division(x, s), by_reciprocal(x, s))


def test_quotients_at_and_beside_every_half_integer():
    rng = np.random.default_rng(1)
    scales = np.float32(np.float16(rng.uniform(1e-4, 3.0, 400)))
    for s in scales:
        for k in range(-1, 17):
            target = np.float32(k + 0.5)
            x0 = np.multiply(target, s, dtype=np.float32)
            xs = [x0]
            up, down = x0, x0
            for _ in range(6):   # neighbouring fp32 values of x: quotients just above / below k + 0.5
                up = np.nextafter(up, np.float32(np.inf), dtype=np.float32)
                down = np.nextafter(down, np.float32(-np.inf), dtype=np.float32)
                xs += [up, down]
            x = np.array(xs, dtype=np.float32)
            assert np.array_equal(by_division(x, s), by_reciprocal(x, s)), (s, k)


def test_clamped_range_and_signs():
    s = np.float32(np.float16(0.37))
    x = np.linspace(-40, 40, 20001, dtype=np.float32) * s
    assert np.array_equal(by_division(x, s), by_reciprocal(x, s))
