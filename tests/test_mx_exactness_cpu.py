"""The arithmetic behind the exact max-pool logits (DraftAttention2 Eq. 3, the
max-pool branch of the draft map), checked on the CPU.

The draft defines a logit as an fp64 fma chain over the channels in ascending
order.  The max-pool descriptors are channel maxima of bf16 inputs, hence bf16
values.  The tensor-core path rests on three facts, checked here with exact
rational arithmetic (no GPU, no package code):

1. a bf16 value with exponent E in a row whose smallest nonzero exponent is e0
   and whose span E - e0 is at most 13 is N * 2^(e0 - 7) with an integer
   |N| < 2^21, and N = 2^14 h + 2^7 m + l with h in [-128, 127] and m, l in
   [0, 127] (three int8 operands);
2. the integer dot product T = sum_c N_ac N_bc equals the sum of the nine part
   products grouped into five accumulators of equal weight
   (2^28, 2^21, 2^14, 2^7, 1), each of which fits an s32 accumulator;
3. for two such rows every partial sum of the fp64 fma chain is an integer
   multiple of 2^(e0a + e0b - 14) below 2^53 of those units, so the chain is
   exact and equals T * 2^(e0a + e0b - 14).
"""
import math
import random
from fractions import Fraction

import numpy as np
import pytest

SPAN = 13


def bf16_value(sign, exp, mant7):
    # normal bf16: (1 + mant7 / 128) * 2^exp
    return (-1) ** sign * (128 + mant7) * 2.0 ** (exp - 7)


def random_row(rng, d, e_lo, span, zeros=0.1):
    row = []
    for _ in range(d):
        if rng.random() < zeros:
            row.append(0.0)
            continue
        e = rng.randint(e_lo, e_lo + span)
        row.append(bf16_value(rng.randint(0, 1), e, rng.randint(0, 127)))
    return row


def exponent(x):
    # exponent E of a nonzero normal value: |x| in [2^E, 2^(E+1))
    return math.frexp(abs(x))[1] - 1


def integer_row(row):
    es = [exponent(x) for x in row if x != 0.0]
    e0 = min(es) if es else 0
    N = []
    for x in row:
        if x == 0.0:
            N.append(0)
            continue
        q = Fraction(x) / Fraction(2) ** (e0 - 7)
        assert q.denominator == 1
        N.append(int(q))
    return N, e0


def split3(n):
    h = n >> 14  # floor
    rest = n - (h << 14)
    return h, rest >> 7, rest & 127


def fma_exact(x, y, z):
    # correctly rounded x * y + z (CPython's int / int true division rounds correctly)
    v = Fraction(x) * Fraction(y) + Fraction(z)
    return v.numerator / v.denominator


@pytest.mark.parametrize("d", [64, 128])
def test_split_and_accumulators(d):
    rng = random.Random(7 + d)
    for _ in range(20):
        row_a = random_row(rng, d, rng.randint(-20, 5), rng.randint(0, SPAN))
        row_b = random_row(rng, d, rng.randint(-20, 5), rng.randint(0, SPAN))
        Na, _ = integer_row(row_a)
        Nb, _ = integer_row(row_b)
        for n in Na + Nb:
            assert abs(n) < 1 << 21
            h, m, l = split3(n)
            assert -128 <= h <= 127 and 0 <= m <= 127 and 0 <= l <= 127
            assert (h << 14) + (m << 7) + l == n
        acc = [0] * 5  # weights 2^(7 (4 - q)), q = qa + qb
        for a, b in zip(Na, Nb):
            pa, pb = split3(a), split3(b)
            for qa in range(3):
                for qb in range(3):
                    acc[qa + qb] += pa[qa] * pb[qb]
        for q in range(5):
            assert -(1 << 31) <= acc[q] < 1 << 31  # an s32 accumulator holds each class
        T = sum(acc[q] << (7 * (4 - q)) for q in range(5))
        assert T == sum(a * b for a, b in zip(Na, Nb))
        assert abs(T) < 1 << 49


@pytest.mark.parametrize("d", [64, 128])
def test_fp64_chain_is_exact_within_the_span(d):
    rng = random.Random(11 + d)
    rd = 1.0 / math.sqrt(d)
    for _ in range(12):
        row_a = random_row(rng, d, rng.randint(-30, 10), rng.randint(0, SPAN))
        row_b = random_row(rng, d, rng.randint(-30, 10), rng.randint(0, SPAN))
        acc = 0.0
        for a, b in zip(row_a, row_b):
            acc = fma_exact(a, b, acc)
        exact = sum(Fraction(a) * Fraction(b) for a, b in zip(row_a, row_b))
        assert Fraction(acc) == exact
        Na, e0a = integer_row(row_a)
        Nb, e0b = integer_row(row_b)
        T = sum(a * b for a, b in zip(Na, Nb))
        via_T = float(T) * 2.0 ** (e0a + e0b - 14)  # exact: |T| < 2^49
        assert via_T == acc
        # the logit: one rounding of the exact value times 1/sqrt(d) on both sides
        assert np.float64(via_T) * np.float64(rd) == np.float64(acc) * np.float64(rd)


def test_chain_can_round_outside_the_span():
    # beyond the range the chain is not exact in general: the fp64 fallback
    # (the defining order) is then required, which the kernel takes
    big, tiny = 2.0 ** 60, 2.0 ** -60
    row_a = [big, tiny, -big]
    row_b = [1.0, 1.0, 1.0]
    acc = 0.0
    for a, b in zip(row_a, row_b):
        acc = fma_exact(a, b, acc)
    exact = sum(Fraction(a) * Fraction(b) for a, b in zip(row_a, row_b))
    assert Fraction(acc) != exact
