"""q // H by one 32-bit multiply-high and a shift (the rows kernel's (token,
head) split for 32-bit row indices): with 2^(s-1) < H <= 2^s and
M = ceil(2^(31+s) / H), (q * M) >> (31 + s) == q // H for 0 <= q < 2^31
(Granlund and Montgomery, PLDI 1994).  Checked here, on the host, at the
start and the end of the range for every head count up to 4096 and for a
sample of larger ones up to the 65536 limit."""

import numpy as np


def _constants(H: int):
    s = (H - 1).bit_length()
    return ((1 << (31 + s)) + H - 1) // H, s


def test_multiply_high_division_is_exact():
    q = np.concatenate([np.arange(0, 8192, dtype=np.uint64),
                        np.uint64(2 ** 31 - 1) - np.arange(0, 8192, dtype=np.uint64)])
    rng = np.random.default_rng(3)
    heads = list(range(2, 4097)) + sorted(set(int(h) for h in rng.integers(4097, 65537, 400))) + [65535, 65536]
    for H in heads:
        M, s = _constants(H)
        assert M < 2 ** 32
        # multiples of H and their neighbours near the top of the range
        top = (np.uint64(2 ** 31 - 1) // np.uint64(H)) * np.uint64(H)
        qq = np.concatenate([q, top - np.arange(0, 3, dtype=np.uint64), top + np.arange(0, 3, dtype=np.uint64)])
        qq = qq[qq < 2 ** 31]
        got = ((qq * np.uint64(M)) >> np.uint64(32)) >> np.uint64(s - 1)
        assert np.array_equal(got, qq // np.uint64(H)), H


def test_a_truncated_constant_breaks_it():
    """floor instead of ceil in M misses every multiple of H (H not a power
    of two): the check has teeth."""
    H = 27
    _, s = _constants(H)
    M = (1 << (31 + s)) // H
    q = np.arange(1, 100, dtype=np.uint64) * np.uint64(H)
    got = ((q * np.uint64(M)) >> np.uint64(32)) >> np.uint64(s - 1)
    assert np.all(got == q // np.uint64(H) - np.uint64(1))
