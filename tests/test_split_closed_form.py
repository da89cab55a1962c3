"""Host-side check of the combine's closed form for the stream-K split.

The decode kernels give persistent CTA c the work units
[floor(c*U/N), floor((c+1)*U/N)); the combine finds the CTA holding unit u as
((u+1)*N - 1) // U (csrc/decode_gqa.cu, owner_cta), so that a segment's pieces
are the CTAs from the owner of its first unit to the owner of its last.  This
compares that closed form with the split itself, by brute force.
"""
import random

import pytest


def owner_closed_form(u, n, total):
    return ((u + 1) * n - 1) // total


def owners_by_split(n, total):
    own = [None] * total
    for c in range(n):
        for u in range(c * total // n, (c + 1) * total // n):
            own[u] = c
    return own


@pytest.mark.parametrize("total", range(1, 80))
def test_closed_form_matches_the_split_small(total):
    for n in range(1, min(total, 60) + 1):           # the kernels use N = min(CTAs, U)
        own = owners_by_split(n, total)
        assert all(owner_closed_form(u, n, total) == own[u] for u in range(total)), (n, total)


def test_closed_form_matches_the_split_random_large():
    rng = random.Random(7)
    for _ in range(200):
        total = rng.randrange(80, 400_000)
        n = rng.randrange(1, min(total, 5_000) + 1)
        for _ in range(50):
            c = rng.randrange(n)
            lo, hi = c * total // n, (c + 1) * total // n
            for u in {lo, hi - 1, (lo + hi) // 2}:
                if lo <= u < hi:
                    assert owner_closed_form(u, n, total) == c, (u, n, total)


def test_segment_pieces_are_contiguous_ctas():
    # a segment [S, E) is covered by CTAs owner(S) .. owner(E-1), each holding a nonempty part
    rng = random.Random(3)
    for _ in range(300):
        total = rng.randrange(1, 5_000)
        n = rng.randrange(1, min(total, 300) + 1)
        s = rng.randrange(total)
        e = rng.randrange(s + 1, total + 1)
        first, last = owner_closed_form(s, n, total), owner_closed_form(e - 1, n, total)
        for c in range(first, last + 1):
            lo, hi = max(s, c * total // n), min(e, (c + 1) * total // n)
            assert lo < hi, (c, s, e, n, total)
