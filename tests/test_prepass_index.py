"""Host-side check of the multiply-high division the prepass kernels use for
the head index of a 16-byte vector: with m = ceil(2^64 / d) (m = 0 for d = 1),
floor(n m / 2^64) = floor(n / d) for every n < 2^32 and d < 2^32.  Checked on
the divisors the kernels meet (vectors per head row for D = 8 .. 1024 and head
counts up to 4096) at the ends of the range and on random numerators."""
import random


def magic(d):
    return 0 if d <= 1 else (2**64 - 1) // d + 1


def div(n, m):
    return n if m == 0 else (n * m) >> 64


def test_multiply_high_division_is_exact():
    rng = random.Random(5)
    divisors = sorted({d for D in range(8, 1025, 8) for d in (D // 8, D // 4)} | set(range(1, 4097)))
    for d in divisors:
        m = magic(d)
        ns = [0, 1, d - 1, d, d + 1, 2**32 - 1, 2**32 - 2, (2**32 - 1) // d * d, (2**32 - 1) // d * d - 1]
        ns += [rng.randrange(2**32) for _ in range(40)]
        for n in ns:
            if 0 <= n < 2**32:
                assert div(n, m) == n // d, (n, d)


def test_head_index_of_a_vector():
    # vec_head: q = vi // vph, head = q - H * (q // H)
    for H, vph in ((32, 16), (8, 16), (16, 24), (3, 5), (4096, 128), (1, 1)):
        mv, mh = magic(vph), magic(H)
        for vi in list(range(0, 3 * H * vph)) + [2**31 + 7, 2**32 - 1]:
            q = div(vi, mv)
            assert q - H * div(q, mh) == (vi // vph) % H
