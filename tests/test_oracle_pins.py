"""The fp64 oracle against its pins (CPU only)."""
import numpy as np
import pytest

import oracle
import oracle_pins


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check(oracle.load())


def test_paged_to_cache_round_trip():
    """A cache cut into pages under a random page permutation and gathered
    back through the table is the cache again; an identity table on a pool
    laid out sequence by sequence is a plain reshape; ids outside the pool
    and rows past the length read as zero."""
    rng = np.random.default_rng(5)
    B, n_kv, P, ps, d = 3, 2, 5, 4, 3
    cache = rng.standard_normal((B, n_kv, P * ps, d))
    perm = rng.permutation(B * P)                  # logical page (b, p) -> pool page perm[b*P+p]
    pool = np.zeros((B * P, ps, n_kv, d))
    for b in range(B):
        for p in range(P):
            pool[perm[b * P + p]] = cache[b, :, p * ps:(p + 1) * ps, :].transpose(1, 0, 2)
    table = perm.reshape(B, P)
    full = [P * ps] * B
    assert np.array_equal(oracle.paged_to_cache(pool, table, full), cache)
    # identity table: pool page b*P+p holds tokens p*ps .. of sequence b
    ident = np.arange(B * P).reshape(B, P)
    pool2 = cache.reshape(B, n_kv, P, ps, d).transpose(0, 2, 3, 1, 4).reshape(B * P, ps, n_kv, d)
    assert np.array_equal(oracle.paged_to_cache(pool2, ident, full), cache)
    # a length of 6 keeps rows 0..5; an id past the pool reads zeros
    t2 = table.copy()
    t2[1, 0] = B * P + 3
    got = oracle.paged_to_cache(pool, t2, [6, P * ps, 0])
    assert np.array_equal(got[0, :, :6], cache[0, :, :6]) and not got[0, :, 6:].any()
    assert not got[1, :, :ps].any() and np.array_equal(got[1, :, ps:], cache[1, :, ps:])
    assert not got[2].any()
