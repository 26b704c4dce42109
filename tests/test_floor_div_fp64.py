"""The decode kernels find the owner of an item, floor(a / b) with 0 <= a < 2^53
and 1 <= b < 2^31, through one IEEE fp64 division and a floor (lora_tile.cuh:
floor_div_small) where the quotient is below 2^21. Python floats are IEEE
doubles and `/` rounds to nearest, so the claim is checked here against exact
integer division, on the cases closest to an integer from either side."""
import math
import random

import pytest


def _cases():
    rng = random.Random(7)
    # b up to 2^31 - 1, quotients up to 2^21 - 1, a = k b + d with d near 0 and near b
    for _ in range(20000):
        b = rng.randrange(1, 1 << 31)
        k = rng.randrange(0, 1 << 21)
        for d in (0, 1, 2, b - 1, b - 2, rng.randrange(0, b)):
            a = k * b + d
            if 0 <= d < b and a < (1 << 53):
                yield a, b
    # the largest quotients with the largest divisors
    for b in ((1 << 31) - 1, (1 << 31) - 2, 1 << 30, 3, 1):
        for k in ((1 << 21) - 1, (1 << 21) - 2, 1 << 20):
            for d in (0, 1, b - 1):
                a = k * b + d
                if 0 <= d < b and a < (1 << 53):
                    yield a, b


def test_floor_of_rounded_quotient_is_exact():
    n = 0
    for a, b in _cases():
        assert math.floor(a / b) == a // b, (a, b)
        n += 1
    assert n > 100000


@pytest.mark.parametrize("n_items,n_units", [(11008, 296), (1376, 296), (44032, 2368), (2**31 - 1, 2368)])
def test_owner_formula_matches_ranges(n_items, n_units):
    # owner(i) = floor(((i + 1) n_units - 1) / n_items) is the unit u whose range
    # [u n_items / n_units, (u + 1) n_items / n_units) holds item i
    rng = random.Random(n_items)
    items = [0, n_items - 1] + [rng.randrange(n_items) for _ in range(2000)]
    for i in items:
        u = math.floor(((i + 1) * n_units - 1) / n_items)
        assert u * n_items // n_units <= i < (u + 1) * n_items // n_units, (i, u)
